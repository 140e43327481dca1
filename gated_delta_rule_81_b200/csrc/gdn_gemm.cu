// Dense bf16 projections around the mixer: C = A B^T with fp32 accumulation.
//
// Agnes-3.0-Flash model card, "Architecture" table: hidden size 5120, and the row
// "Delta-rule layers" (16 key heads / 48 value heads, head dim 128).  The mixer's
// inputs (q, k, v, the output gate z and the per-head gate logits a, b) come from
// the hidden state through one input projection, and its 48 x 128 outputs go back
// to the hidden size through one output projection.  Both are plain matrix products,
// which this file computes on the tensor cores.
//
// One persistent CTA per SM walks 128 x BN output tiles (M fastest, so the CTAs
// running at the same time share B tiles through L2).  Per tile and 64-wide K step,
// warp 0 lane 0 loads the A (128 x 64) and B (BN x 64) boxes with TMA (128-byte
// swizzle, zero fill past the matrix edges) into a ring of stages; warp 1 lane 0
// issues four tcgen05.mma (M 128, N BN, K 16) per step into one of two fp32
// accumulators in tensor memory (columns 0 and 256); warps 2-5 read the other accumulator
// (thread = row, lane quarter = warp % 4), round to bf16 and store, so each tile's
// epilogue overlaps the next tile's products.  BN (256, 224, 192 or 160) is chosen
// per shape (gemm_tile_width) so that the last round of tiles is not mostly idle.  Every wait is bounded: a
// stuck wait sets error bit 1 and the CTA unwinds (draining its copies and products).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_kernels.cuh"

namespace gdn {

namespace {

constexpr int kGemmBM = 128, kGemmBK = 64;
constexpr int kGemmABytes = kGemmBM * kGemmBK * 2;  // 16 KiB
constexpr int kGemmThreads = 192;  // warp 0: TMA, warp 1: MMA, warps 2-5: epilogue
constexpr int kGemmEpiWarps = 4;
constexpr int kGemmSmemBudget = 220 * 1024;

template <int BN>
struct GemmTile {
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStageBytes = kGemmABytes + kBBytes;
  static constexpr int kStages = (kGemmSmemBudget - 1024) / kStageBytes > 6 ? 6 : (kGemmSmemBudget - 1024) / kStageBytes;
  static constexpr int kSmem = kStages * kStageBytes + 1024;
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "tile width");
};

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n;
  bf16* C;
  long long ldc;
  int* err;
};

__device__ __forceinline__ uint8_t* gemm_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 2-D tiled TMA load of the box at (x = column, y = row) into shared memory, completing on bar
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                     GemmParams g) {
  constexpr int kGemmBN = BN, kGemmStages = GemmTile<BN>::kStages, kGemmStageBytes = GemmTile<BN>::kStageBytes;
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* sm = gemm_align1024(gemm_smem_raw);
  __shared__ uint64_t full[kGemmStages], empty[kGemmStages], acc_full[2], acc_empty[2], drain_b;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Abort ab{g.err, &abort_s};
  if (threadIdx.x == 0) {
    abort_s = 0;
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kGemmEpiWarps);
    }
    mbar_init(&drain_b, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc<512>(&tmem_base_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;
  const int n_tiles = g.tiles_m * g.tiles_n;
  const int k_steps = g.K / kGemmBK;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      long long it = 0;
      for (int t = blockIdx.x; t < n_tiles && !ab.raised(); t += gridDim.x) {
        const int m0 = (t % g.tiles_m) * kGemmBM, n0 = (t / g.tiles_m) * kGemmBN;
        bool ok = true;
        for (int kk = 0; kk < k_steps; ++kk, ++it) {
          const int s = static_cast<int>(it % kGemmStages);
          const long long use = it / kGemmStages;
          if (use > 0 && !mbar_wait(&empty[s], static_cast<uint32_t>((use - 1) & 1), ab)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kGemmStageBytes);
          uint8_t* st = sm + s * kGemmStageBytes;
          tma_load_2d(st, &tma_a, kk * kGemmBK, m0, &full[s]);
          tma_load_2d(st + kGemmABytes, &tma_b, kk * kGemmBK, n0, &full[s]);
        }
        if (!ok) break;
      }
      // loads still in flight (only after an abort) land before the CTA exits
      int drain_flag = 0;
      const Abort drain{nullptr, &drain_flag};
      for (int s = 0; s < kGemmStages; ++s) {
        const long long uses = it > s ? (it - 1 - s) / kGemmStages + 1 : 0;  // loads issued into stage s
        if (uses > 0) mbar_wait(&full[s], static_cast<uint32_t>((uses - 1) & 1), drain);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16(kGemmBM, kGemmBN, false, false);
      long long it = 0;
      int tile_i = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tile_i) {
        const int b = tile_i & 1, buse = tile_i >> 1;
        if (buse > 0 && !mbar_wait(&acc_empty[b], (buse - 1) & 1, ab)) break;
        tc_fence_after();
        const uint32_t d = tbase + static_cast<uint32_t>(b * 256);
        for (int kk = 0; kk < k_steps; ++kk, ++it) {
          const int s = static_cast<int>(it % kGemmStages);
          if (!mbar_wait(&full[s], static_cast<uint32_t>((it / kGemmStages) & 1), ab)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = smem_u32(sm + s * kGemmStageBytes), b_s = a_s + kGemmABytes;
#pragma unroll
          for (int ks = 0; ks < kGemmBK / 16; ++ks)
            umma_bf16(d, smem_desc(a_s + ks * 32u, 16, 1024, Swz::k128), smem_desc(b_s + ks * 32u, 16, 1024, Swz::k128),
                      idesc, kk > 0 || ks > 0);
          umma_commit(&empty[s]);  // the stage is free once these products have read it
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      // every product issued has completed before tensor memory is released
      umma_commit(&drain_b);
      int drain_flag = 0;
      const Abort drain{nullptr, &drain_flag};
      mbar_wait(&drain_b, 0, drain);
    }
  } else {
    // ------------------------------------------------ epilogue: thread = output row
    const int q = warp & 3;
    int tile_i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tile_i) {
      const int b = tile_i & 1;
      if (!mbar_wait_warp(&acc_full[b], (tile_i >> 1) & 1, ab, false, 32)) break;
      tc_fence_after();
      const int m0 = (t % g.tiles_m) * kGemmBM, n0 = (t / g.tiles_m) * kGemmBN;
      const int row = m0 + 32 * q + lane;
      bf16* crow = g.C + static_cast<long long>(row) * g.ldc + n0;
#pragma unroll 1
      for (int c = 0; c < kGemmBN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem_addr(tbase, 32 * q, static_cast<uint32_t>(b * 256 + 32 * c)), v);
        tmem_wait_ld();
        const int col = n0 + 32 * c;
        if (row < g.M && col < g.N) {
          if (col + 32 <= g.N) {
            uint4* dst = reinterpret_cast<uint4*>(crow + 32 * c);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                  pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (col + e < g.N) crow[32 * c + e] = __float2bfloat16(v[e]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc<512>(tbase);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// K-major bf16 matrix [rows][ld] (first `cols` columns used) as 64 x box_rows boxes, 128-byte swizzle
bool encode_kmajor(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, long long rows,
                   long long cols, long long ld, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kGemmBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace {

template <int BN>
cudaError_t launch_gemm_tile(PFN_cuTensorMapEncodeTiled_v12000 enc, const bf16* A, long long lda, const bf16* B,
                             long long ldb, bf16* C, long long ldc, int M, int N, int K, int* err, int n_sm,
                             cudaStream_t stream) {
  CUtensorMap ta, tb;
  if (!encode_kmajor(enc, &ta, A, M, K, lda, kGemmBM) || !encode_kmajor(enc, &tb, B, N, K, ldb, BN))
    return cudaErrorInvalidValue;
  GemmParams g;
  g.M = M;
  g.N = N;
  g.K = K;
  g.tiles_m = (M + kGemmBM - 1) / kGemmBM;
  g.tiles_n = (N + BN - 1) / BN;
  g.C = C;
  g.ldc = ldc;
  g.err = err;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GemmTile<BN>::kSmem);
  if (e != cudaSuccess) return e;
  const long long n_tiles = static_cast<long long>(g.tiles_m) * g.tiles_n;
  const unsigned grid = static_cast<unsigned>(n_tiles < n_sm ? n_tiles : n_sm);
  gemm_bf16_kernel<BN><<<grid, kGemmThreads, GemmTile<BN>::kSmem, stream>>>(ta, tb, g);
  return cudaGetLastError();
}

}  // namespace

// The tile width with the least time in its slowest CTA: rounds of tiles per SM times a
// tile's time, which measures as growing with width + 512 (the A box and the per-step
// hand-offs cost the same at every width); ties go to the wider tile.  At T = 4096 this
// picks 256 for the input projection (N = 16480) and 224 for the output projection
// (N = 5120: 5 rounds of 736 tiles instead of 5 of 640, the last one 32% full).
int gemm_tile_width(int M, int N, int n_sm) {
  static const int kWidths[] = {256, 224, 192, 160};
  int best = 256;
  long long best_cost = -1;
  const long long tiles_m = (M + kGemmBM - 1) / kGemmBM;
  for (int bn : kWidths) {
    const long long tiles = tiles_m * ((N + bn - 1) / bn);
    const long long cost = (tiles + n_sm - 1) / n_sm * (bn + 512);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// ============================================================ weight-streaming product (few rows)
//
// With a handful of rows of A (a decode step: one or a few tokens per sequence) the product is
// bound by reading B, the weights, from HBM once; a 128-row tensor-core tile would be almost
// empty and its few tiles would leave most SMs idle.  One warp takes kGemvCols rows of B (output
// columns): A's rows sit in shared memory as fp32, each lane walks 16-byte pieces of its B rows
// (several loads in flight per lane), multiplies them into fp32 sums per (row of A, column), and
// the warp adds its lanes' sums with shuffles in a fixed order.  One bf16 rounding per output.
constexpr int kGemvThreads = 256;
constexpr int kGemvCols = 2;                                   // B rows (output columns) per warp
constexpr int kGemvColsPerCta = kGemvCols * kGemvThreads / 32;

template <int MR>
__global__ void __launch_bounds__(kGemvThreads) gemv_bf16_kernel(const bf16* A, long long lda, const bf16* B,
                                                                 long long ldb, bf16* C, long long ldc, int N, int K) {
  extern __shared__ float4 gemv_x[];  // [MR][K / 4] fp32
  const int kv = K / 8;               // 16-byte pieces per row (K is a multiple of 64)
  for (int i = threadIdx.x; i < MR * kv; i += kGemvThreads) {
    const int m = i / kv, c = i - m * kv;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(A + m * lda) + c);
    gemv_x[m * 2 * kv + 2 * c] = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    gemv_x[m * 2 * kv + 2 * c + 1] = make_float4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w));
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long n0 = static_cast<long long>(blockIdx.x) * kGemvColsPerCta + warp * kGemvCols;
  if (n0 >= N) return;
  const uint4* brow[kGemvCols];
#pragma unroll
  for (int r = 0; r < kGemvCols; ++r)
    brow[r] = reinterpret_cast<const uint4*>(B + (n0 + r < N ? n0 + r : n0) * ldb);
  float acc[kGemvCols][MR];
#pragma unroll
  for (int r = 0; r < kGemvCols; ++r)
#pragma unroll
    for (int m = 0; m < MR; ++m) acc[r][m] = 0.f;
#pragma unroll 4
  for (int c = lane; c < kv; c += 32) {
    uint4 w[kGemvCols];
#pragma unroll
    for (int r = 0; r < kGemvCols; ++r) w[r] = __ldcs(brow[r] + c);  // read once: evict first
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const float4 x0 = gemv_x[m * 2 * kv + 2 * c], x1 = gemv_x[m * 2 * kv + 2 * c + 1];
#pragma unroll
      for (int r = 0; r < kGemvCols; ++r) {
        float a = acc[r][m];
        a = fmaf(bf16_lo(w[r].x), x0.x, a);
        a = fmaf(bf16_hi(w[r].x), x0.y, a);
        a = fmaf(bf16_lo(w[r].y), x0.z, a);
        a = fmaf(bf16_hi(w[r].y), x0.w, a);
        a = fmaf(bf16_lo(w[r].z), x1.x, a);
        a = fmaf(bf16_hi(w[r].z), x1.y, a);
        a = fmaf(bf16_lo(w[r].w), x1.z, a);
        a = fmaf(bf16_hi(w[r].w), x1.w, a);
        acc[r][m] = a;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kGemvCols; ++r)
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float v = acc[r][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == r * MR + m && n0 + r < N) C[m * ldc + n0 + r] = __float2bfloat16(v);
    }
}

template <int MR>
cudaError_t launch_gemv(const bf16* A, long long lda, const bf16* B, long long ldb, bf16* C, long long ldc, int N,
                        int K, cudaStream_t stream) {
  const int smem = MR * K * 4;
  cudaError_t e = cudaFuncSetAttribute(gemv_bf16_kernel<MR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((N + kGemvColsPerCta - 1) / kGemvColsPerCta);
  gemv_bf16_kernel<MR><<<grid, kGemvThreads, smem, stream>>>(A, lda, B, ldb, C, ldc, N, K);
  return cudaGetLastError();
}

cudaError_t launch_gemm_bf16(const bf16* A, long long lda, const bf16* B, long long ldb, bf16* C, long long ldc,
                             int M, int N, int K, int* err, cudaStream_t stream) {
  // a few rows: stream the weights once (A's rows in shared memory, MR * K * 4 bytes)
  if (M <= kGemvMaxM && static_cast<long long>(M) * K * 4 <= 200 * 1024) {
    switch (M) {
      case 1: return launch_gemv<1>(A, lda, B, ldb, C, ldc, N, K, stream);
      case 2: return launch_gemv<2>(A, lda, B, ldb, C, ldc, N, K, stream);
      case 3: return launch_gemv<3>(A, lda, B, ldb, C, ldc, N, K, stream);
      default: return launch_gemv<4>(A, lda, B, ldb, C, ldc, N, K, stream);
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  switch (gemm_tile_width(M, N, n_sm)) {
    case 224: return launch_gemm_tile<224>(enc, A, lda, B, ldb, C, ldc, M, N, K, err, n_sm, stream);
    case 192: return launch_gemm_tile<192>(enc, A, lda, B, ldb, C, ldc, M, N, K, err, n_sm, stream);
    case 160: return launch_gemm_tile<160>(enc, A, lda, B, ldb, C, ldc, M, N, K, err, n_sm, stream);
    default: return launch_gemm_tile<256>(enc, A, lda, B, ldb, C, ldc, M, N, K, err, n_sm, stream);
  }
}

}  // namespace gdn
