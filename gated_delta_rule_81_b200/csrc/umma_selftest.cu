// Self-test of the UMMA operand layouts and descriptors used by the mixer
// kernels: one CTA computes D[128 x N] = A[128 x K] * B[N x K]^T with
// tcgen05.mma (bf16 in, fp32 accumulate in TMEM) after staging A and B in
// shared memory in the requested swizzled layout.  Built into its own test
// library (libgdn_selftest.so); the mixer library does not contain it.
#include "gdn_ptx.cuh"

using namespace gdn;

namespace {

// layout codes
constexpr int kKMajor = 0;     // SW128, K-major
constexpr int kMN128 = 1;      // SW128, MN-major (64-wide MN blocks, LBO apart)
constexpr int kMN64 = 2;       // SW64, MN-major (32-wide MN blocks, LBO apart)
constexpr int kTmemA = 3;      // A only: in tensor memory, lane = row m, bf16 pairs along K per column

__device__ __forceinline__ uint32_t operand_off(int layout, int mn, int k, int MN, int K) {
  if (layout == kKMajor) {  // K blocks of 64 elements, each MN rows x 128 B
    return static_cast<uint32_t>((k >> 6) * (MN * 128)) + sw128_off(mn, (k & 63) >> 3) + (k & 7) * 2;
  }
  if (layout == kMN128) {  // MN blocks of 64 elements, each K rows x 128 B
    return static_cast<uint32_t>((mn >> 6) * (K * 128)) + sw128_off(k, (mn & 63) >> 3) + (mn & 7) * 2;
  }
  // 32-wide MN blocks of K rows x 64 B each
  return static_cast<uint32_t>((mn >> 5) * (K * 64)) + sw64_off(k, (mn & 31) >> 3) + (mn & 7) * 2;
}

__device__ __forceinline__ uint64_t operand_desc(int layout, uint32_t base, int ks, int MN, int K) {
  if (layout == kKMajor) {
    uint32_t addr = base + (ks * 16 / 64) * (MN * 128) + ((ks * 16) % 64) * 2;
    return smem_desc(addr, 16, 1024, Swz::k128);
  }
  if (layout == kMN128) return smem_desc(base + ks * 2048, K * 128, 1024, Swz::k128);
  return smem_desc(base + ks * 1024, K * 64, 512, Swz::k64);
}

__global__ void __launch_bounds__(128) umma_selftest_kernel(int a_layout, int b_layout, int N, int K,
                                                            const __nv_bfloat16* __restrict__ A,
                                                            const __nv_bfloat16* __restrict__ B,
                                                            float* __restrict__ D, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                       // 128 x K bf16
  uint8_t* sB = smem + 128 * K * 2;         // N x K bf16
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5;
  Abort ab{err, &abort_flag};

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc<512>(&tmem_base);
  if (a_layout != kTmemA) {
    for (int i = tid; i < 128 * K; i += blockDim.x) {
      int m = i / K, k = i % K;
      *reinterpret_cast<__nv_bfloat16*>(sA + operand_off(a_layout, m, k, 128, K)) = A[i];
    }
  }
  for (int i = tid; i < N * K; i += blockDim.x) {
    int n = i / K, k = i % K;
    *reinterpret_cast<__nv_bfloat16*>(sB + operand_off(b_layout, n, k, N, K)) = B[i];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  if (a_layout == kTmemA) {
    // row m = TMEM lane m, columns 256 + c hold the bf16 pair (A[m][2c], A[m][2c+1]), even k in the low half
    const uint32_t* A32 = reinterpret_cast<const uint32_t*>(A);
    for (int c0 = 0; c0 < K / 2; c0 += 32) {
      uint32_t w[32];
      for (int j = 0; j < 32; ++j) w[j] = A32[(tid * K) / 2 + c0 + j];
      tmem_st32(tmem_addr(tbase, warp * 32, 256 + c0), reinterpret_cast<const float*>(w));
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (tid == 0) {
    uint32_t idesc = idesc_bf16(128, N, a_layout == kMN128 || a_layout == kMN64, b_layout != kKMajor);
    for (int ks = 0; ks < K / 16; ++ks) {
      uint64_t db = operand_desc(b_layout, smem_u32(sB), ks, N, K);
      if (a_layout == kTmemA) {
        umma_bf16_ts(tbase, tbase + 256 + 8 * ks, db, idesc, ks > 0);
      } else {
        uint64_t da = operand_desc(a_layout, smem_u32(sA), ks, 128, K);
        umma_bf16(tbase, da, db, idesc, ks > 0);
      }
    }
    umma_commit(&bar);
  }
  __syncwarp();
  bool ok = mbar_wait(&bar, 0, ab);
  tc_fence_after();
  if (ok) {
    const int row = warp * 32 + (tid & 31);
    for (int c0 = 0; c0 < N; c0 += 32) {
      float v[32];
      tmem_ld32(tmem_addr(tbase, warp * 32, c0), v);
      tmem_wait_ld();
      for (int j = 0; j < 32; ++j) D[row * N + c0 + j] = v[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<512>(tbase);
}

}  // namespace

// D = A * B^T for a 128 x K A and an N x K B (both bf16 row-major, device), fp32 D [128][N].
// a_layout / b_layout: 0 = K-major SW128, 1 = MN-major SW128, 2 = MN-major SW64 (32-wide MN blocks);
// a_layout 3 = A in tensor memory (K <= 256).
// Returns 0 on launch success, -1 on a bad argument, else the CUDA error code.
extern "C" int gdn_selftest_umma(int a_layout, int b_layout, int N, int K, const void* A, const void* B,
                                 float* D, int* err, void* stream) {
  if (K % 64 != 0 || K < 64 || K > 256) return -1;
  if (N % 16 != 0 || N < 16 || N > 256) return -1;
  if (a_layout == 2 || a_layout > 3 || b_layout > 2) return -1;
  if (a_layout == 1 && K % 16 != 0) return -1;
  if (b_layout == 1 && N % 64 != 0) return -1;
  if (b_layout == 2 && N % 32 != 0) return -1;
  size_t smem = static_cast<size_t>(128 + N) * K * 2 + 1024;
  cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  umma_selftest_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      a_layout, b_layout, N, K, static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), D, err);
  return static_cast<int>(cudaGetLastError());
}
