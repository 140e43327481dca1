// Chunked prefill of the gated-delta-rule mixer on sm_100a.
//
// Method: Agnes-3.0-Flash model card, "Architecture" table, row "Delta-rule
// layers" (16 key / 48 value heads, head dim 128, causal conv kernel 4 in
// front, gated RMS-norm after, fp32 recurrent state) and "Agnes-3.0-Flash
// Deep Dive: A 33B Hybrid-Attention Multimodal Model", section "Feed-Forward
// and Positional Encoding", paragraph on the Gated Delta Rule (erase-then-write
// under a forget gate).  Recurrence: S_t = a_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T,
// o_t = S_t q_t, evaluated 64 tokens at a time in its chunkwise (UT-transform)
// form.  Inside a chunk that starts from state S (d_v x d_k), with G the
// inclusive cumulative sum of g = log a, gamma_i = e^{G_i}:
//   A_ij = b_i e^{G_i - G_j} (k_i . k_j) (j < i),   T = (I + A)^{-1},
//   T~ = T diag(b),   P_ij = e^{G_i - G_j} (q_i . k_j) (j <= i),
//   R = V - diag(gamma) K S^T,   U = T~ R,   O = diag(gamma) Q S^T + P T~ R,
//   S^T <- gamma_C S^T + K^T diag(e^{G_C - G_j}) U.
//
// Two kernels (plus two small helpers):
//   prep (one CTA per chunk x key head, all chunks in parallel): conv + SiLU +
//     L2-norm front end, gates, [Q;K] K^T on tcgen05, the fp32 blocked
//     triangular solve, and [P;I] T~ on tcgen05.  It writes the chunk's
//     operand images to the workspace.
//   scan (one CTA, or a cluster of 2 or 4 CTAs, per sequence x value head;
//     each CTA owns 128/cluster value rows of the state): walks the chunks in
//     order with S^T resident in tensor memory.  Per chunk three tcgen05 MMAs
//     ([Q;K] S^T, [P T~; T~] R, K^T U) and the gated RMS-norm epilogue.
#include "gdn_kernels.cuh"

namespace gdn {

namespace {

constexpr int kDevErrBadSeqlens = 4;
constexpr int kMaxOrdered = 8192;  // sequences reordered longest-first for the scan
constexpr unsigned kBackoffNs = 64;  // poll back-off of the producer and output warps

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ long long seq_start(const PrefillParams& p, int n) {
  return p.cu ? static_cast<long long>(p.cu[n]) : static_cast<long long>(n) * p.T_uniform;
}

__device__ __forceinline__ long long chunk_base_of(const PrefillParams& p, int n) {
  return p.chunk_base ? static_cast<long long>(p.chunk_base[n])
                      : static_cast<long long>(n) * ((p.T_uniform + kChunk - 1) / kChunk);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Named barrier over `nthreads` threads that also ORs a per-thread predicate:
// every participant gets the same answer.  The non-aligned form, so the lanes of
// a warp may arrive at different times (one lane may still be issuing MMAs).
__device__ __forceinline__ bool bar_sync_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float ld_shared_remote(const float* p, uint32_t cta) {
  uint32_t local = smem_u32(p), remote;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(cta));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// unpack 8 bf16 from a uint4
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// ============================================================ helpers

// chunk_base[n] = sum_{m<n} ceil(L_m / 64) from the device cu_seqlens; checks
// that the device copy is valid (cu[0] = 0, non-decreasing) and agrees with the
// host copy in its number of chunks and its total number of tokens.
__global__ void __launch_bounds__(1024) setup_kernel(PrefillParams p) {
  __shared__ long long part[1024];
  __shared__ int bad_s;
  const int tid = threadIdx.x;
  if (tid == 0) bad_s = (p.cu[0] != 0) || (static_cast<long long>(p.cu[p.N]) != p.T_total);
  __syncthreads();
  const int per = (p.N + 1023) / 1024;
  const int n0 = min(tid * per, p.N), n1 = min(n0 + per, p.N);
  long long acc = 0;
  int bad = 0;
  for (int n = n0; n < n1; ++n) {
    const int L = p.cu[n + 1] - p.cu[n];
    if (L < 0) bad = 1;
    acc += L > 0 ? (L + kChunk - 1) / kChunk : 0;
  }
  if (bad) atomicOr(&bad_s, 1);
  part[tid] = acc;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan
    const long long v = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  long long base = part[tid] - acc;
  for (int n = n0; n < n1; ++n) {
    p.chunk_base[n] = static_cast<int>(base);
    const int L = p.cu[n + 1] - p.cu[n];
    base += L > 0 ? (L + kChunk - 1) / kChunk : 0;
  }
  if (tid == 1023) {
    p.chunk_base[p.N] = static_cast<int>(part[1023]);
    if (part[1023] != p.n_chunks) atomicOr(&bad_s, 1);
  }
  // scan order: longest sequence first (ties by index), so the longest chains start
  // in the first wave; beyond kMaxOrdered sequences the pack order is kept
  if (p.N <= kMaxOrdered) {
    for (int nn = tid; nn < p.N; nn += 1024) {
      const int Ln = p.cu[nn + 1] - p.cu[nn];
      int rank = 0;
      for (int m = 0; m < p.N; ++m) {
        const int Lm = p.cu[m + 1] - p.cu[m];
        rank += (Lm > Ln || (Lm == Ln && m < nn)) ? 1 : 0;
      }
      p.seq_order[rank] = nn;
    }
  }
  __syncthreads();
  if (tid == 0) {
    *p.ws_flag = bad_s;
    if (bad_s && p.err) atomicOr(p.err, kDevErrBadSeqlens);
  }
}

// raw (pre-conv) value of conv channel c at token tau (tau inside the packed batch)
__device__ __forceinline__ bf16 raw_channel(const PrefillParams& p, long long tau, long long c) {
  const long long qk = static_cast<long long>(p.H_k) * kD;
  if (c < qk) return p.q[tau * p.sq + c];
  if (c < 2 * qk) return p.k[tau * p.sk + (c - qk)];
  return p.v[tau * p.sv + (c - 2 * qk)];
}

// conv_out[n][j][c] = raw channel c at token end-3+j (history from conv_in before the start)
__global__ void conv_out_kernel(PrefillParams p) {
  const int n = blockIdx.y;
  const long long C_conv = static_cast<long long>(2 * p.H_k + p.H_v) * kD;
  const long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= C_conv) return;
  if (p.cu && *p.ws_flag) return;
  const long long s = seq_start(p, n), e = seq_start(p, n + 1);
  for (int j = 0; j < 3; ++j) {
    const long long tau = e - 3 + j;
    bf16 val;
    if (tau >= s) val = raw_channel(p, tau, c);
    else if (p.conv_in) val = p.conv_in[(static_cast<long long>(n) * 3 + 3 + (tau - s)) * C_conv + c];
    else val = __float2bfloat16(0.f);
    p.conv_out[(static_cast<long long>(n) * 3 + j) * C_conv + c] = val;
  }
}

// ============================================================ prep kernel

constexpr int kPrepThreads = 256;
constexpr int kLdA = 65;                               // fp32 row stride of A in shared memory
constexpr int kLdT = 68;                               // fp32 row stride of T (16-byte aligned rows)
constexpr int kPrepOffQK = 0;                          // [Q;K] image hi, lo    2 x 32768
// After the [Q;K] K^T product has completed, the [Q;K] region is reused by the head loop:
constexpr int kPrepOffTt = kPrepOffQK;                 // T~ image (B) hi, lo   2 x 8192
constexpr int kPrepOffA = kPrepOffTt + 2 * 8192;       // A fp32                64*65*4
constexpr int kPrepOffT = kPrepOffA + 64 * kLdA * 4;   // T fp32                64*68*4
constexpr int kPrepOffM = kPrepOffT + 64 * kLdT * 4;   // block-solve temp      3*256*4
static_assert(kPrepOffM + 3 * 256 * 4 <= 2 * 32768, "head-loop buffers must fit the [Q;K] region");
constexpr int kPrepOffPI = 2 * 32768;                  // [P;I] image hi, lo    2 x 16384
constexpr int kPrepOffG = kPrepOffPI + 2 * 16384;      // G cumsum [8][64]
constexpr int kPrepOffB = kPrepOffG + 8 * 64 * 4;      // beta     [8][64]
constexpr int kPrepOffW = kPrepOffB + 8 * 64 * 4;      // conv weights of the CTA's channels, (2+G)*128*8 B
// dynamic shared memory for G value heads per key head (1 KiB of alignment slack)
__host__ __device__ constexpr int prep_smem_bytes(int G) { return kPrepOffW + (2 + G) * 128 * 8 + 1024; }

// hi = bf16(f), lo = bf16(f - hi) for 8 values
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    h[e] = __bfloat162float(__float2bfloat16(f[e]));
    l[e] = f[e] - h[e];
  }
  hi = pack8(h);
  lo = pack8(l);
}

// Conv (4 taps) + SiLU of 32 consecutive channels of one token.
//   src: the token-0 address of the group's first channel; rows before the
//   sequence start come from conv_in (or are zero).  wsm: the 32 channels'
//   weights in shared memory, 16 x uint4 (channels 2u, 2u+1; taps 0..3 each).
//   All 16 input loads are issued before any arithmetic.
__device__ __forceinline__ void conv32(const PrefillParams& p, const bf16* src, long long src_stride,
                                       long long s, long long t, int n, long long conv_chan0, const uint4* wsm,
                                       float* y) {
  const long long C_conv = static_cast<long long>(2 * p.H_k + p.H_v) * kD;
  uint4 xin[kTaps][4];
#pragma unroll
  for (int j = 0; j < kTaps; ++j) {
    const long long tau = t - (kTaps - 1) + j;
    const uint4* row = nullptr;
    if (tau >= s) row = reinterpret_cast<const uint4*>(src + tau * src_stride);
    else if (p.conv_in)
      row = reinterpret_cast<const uint4*>(p.conv_in + (static_cast<long long>(n) * 3 + 3 + (tau - s)) * C_conv +
                                           conv_chan0);
#pragma unroll
    for (int g = 0; g < 4; ++g) xin[j][g] = row ? __ldg(row + g) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float x[kTaps][8];
#pragma unroll
    for (int j = 0; j < kTaps; ++j) unpack8(xin[j][g], x[j]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // channel pair 8g + 2u, 8g + 2u + 1
      const uint4 w = wsm[4 * g + u];
      const int e0 = 2 * u, e1 = 2 * u + 1;
      float a0 = bf16_lo(w.x) * x[0][e0];
      a0 = fmaf(bf16_hi(w.x), x[1][e0], a0);
      a0 = fmaf(bf16_lo(w.y), x[2][e0], a0);
      a0 = fmaf(bf16_hi(w.y), x[3][e0], a0);
      float a1 = bf16_lo(w.z) * x[0][e1];
      a1 = fmaf(bf16_hi(w.z), x[1][e1], a1);
      a1 = fmaf(bf16_lo(w.w), x[2][e1], a1);
      a1 = fmaf(bf16_hi(w.w), x[3][e1], a1);
      y[8 * g + e0] = silu_fast(a0);
      y[8 * g + e1] = silu_fast(a1);
    }
  }
}

// One block diagonal of the blocked inverse: for blocks (I, J = I - d),
//   M = sum_{K=J}^{I-1} A_IK T_KJ,   T_IJ = -T_II M
// with 16x16 blocks; each thread computes four adjacent columns of one row.
template <int d>
__device__ __forceinline__ void solve_level(const float* sA, float* sT, float* sM, int tid) {
  constexpr int nb = 4 - d;
  if (tid < nb * 64) {
    const int J = tid >> 6, I = J + d, ii = (tid >> 2) & 15, j4 = (tid & 3) * 4;
    const float* arow = sA + (16 * I + ii) * kLdA + 16 * J;
    const float* tcol = sT + (16 * J) * kLdT + 16 * J + j4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int kk = 0; kk < 16 * d; ++kk) {
      const float a = arow[kk];
      const float4 t = *reinterpret_cast<const float4*>(tcol + kk * kLdT);
      acc.x = fmaf(a, t.x, acc.x);
      acc.y = fmaf(a, t.y, acc.y);
      acc.z = fmaf(a, t.z, acc.z);
      acc.w = fmaf(a, t.w, acc.w);
    }
    *reinterpret_cast<float4*>(sM + (J << 8) + (ii << 4) + j4) = acc;
  }
  __syncthreads();
  if (tid < nb * 64) {
    const int J = tid >> 6, I = J + d, ii = (tid >> 2) & 15, j4 = (tid & 3) * 4;
    const float* trow = sT + (16 * I + ii) * kLdT + 16 * I;
    const float* mcol = sM + (J << 8) + j4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int l = 0; l < 16; ++l) {  // T_II is lower triangular (its upper part is stored as zeros)
      const float a = trow[l];
      const float4 m = *reinterpret_cast<const float4*>(mcol + (l << 4));
      acc.x = fmaf(a, m.x, acc.x);
      acc.y = fmaf(a, m.y, acc.y);
      acc.z = fmaf(a, m.z, acc.z);
      acc.w = fmaf(a, m.w, acc.w);
    }
    *reinterpret_cast<float4*>(sT + (16 * I + ii) * kLdT + 16 * J + j4) = make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
  }
  __syncthreads();
}

// T = (I + A)^{-1} for a 64x64 strictly-lower A (fp32, shared memory), by 16x16
// blocks: diagonal blocks by forward substitution, then the three block
// diagonals below.  All 256 threads.
__device__ void solve_unit_lower(const float* sA, float* sT, float* sM, int tid) {
  if (tid < 64) {
    const int blk = tid >> 4, col = tid & 15;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int l = 0; l + 1 < r; l += 2) {
        acc0 = fmaf(sA[(16 * blk + r) * kLdA + 16 * blk + l], x[l], acc0);
        acc1 = fmaf(sA[(16 * blk + r) * kLdA + 16 * blk + l + 1], x[l + 1], acc1);
      }
      if (r & 1) acc0 = fmaf(sA[(16 * blk + r) * kLdA + 16 * blk + r - 1], x[r - 1], acc0);
      const float acc = acc0 + acc1;
      x[r] = r < col ? 0.f : (r == col ? 1.f : -acc);
      sT[(16 * blk + r) * kLdT + 16 * blk + col] = x[r];
    }
  }
  __syncthreads();
  solve_level<1>(sA, sT, sM, tid);
  solve_level<2>(sA, sT, sM, tid);
  solve_level<3>(sA, sT, sM, tid);
}

// D (+)= A B^T with both operands as hi/lo pairs: A_hi B_hi + A_hi B_lo + A_lo B_hi
__device__ __forceinline__ void umma_split(uint32_t d, uint64_t a_hi, uint64_t a_lo, uint64_t b_hi, uint64_t b_lo,
                                           uint32_t idesc, bool accumulate) {
  umma_bf16(d, a_hi, b_hi, idesc, accumulate);
  umma_bf16(d, a_hi, b_lo, idesc, true);
  umma_bf16(d, a_lo, b_hi, idesc, true);
}

__global__ void __launch_bounds__(kPrepThreads, 2) prep_kernel(PrefillParams p) {
  if (p.cu && *p.ws_flag) return;
  extern __shared__ uint8_t prep_smem_raw[];
  uint8_t* sm = align1024(prep_smem_raw);
  uint8_t* sQK = sm + kPrepOffQK;   // hi at +0, lo at +32768
  uint8_t* sPI = sm + kPrepOffPI;   // hi at +0, lo at +16384
  uint8_t* sTt = sm + kPrepOffTt;   // hi at +0, lo at +8192
  float* sA = reinterpret_cast<float*>(sm + kPrepOffA);
  float* sT = reinterpret_cast<float*>(sm + kPrepOffT);
  float* sM = reinterpret_cast<float*>(sm + kPrepOffM);
  float* sG = reinterpret_cast<float*>(sm + kPrepOffG);
  float* sB = reinterpret_cast<float*>(sm + kPrepOffB);
  uint4* sW = reinterpret_cast<uint4*>(sm + kPrepOffW);  // [(2+G)*128 channels / 2] pairs: q | k | v heads
  __shared__ uint64_t bar[3];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long gc = blockIdx.x;
  const int kh = blockIdx.y;
  const int H_k = p.H_k, H_v = p.H_v, G = H_v / H_k;

  // sequence of this chunk: the largest n with chunk_base(n) <= gc
  int n;
  if (p.chunk_base) {
    int lo = 0, hi = p.N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.chunk_base[mid] <= gc) lo = mid; else hi = mid - 1;
    }
    n = lo;
  } else {
    n = static_cast<int>(gc / ((p.T_uniform + kChunk - 1) / kChunk));
  }
  const long long s = seq_start(p, n), e = seq_start(p, n + 1);
  const long long t0 = s + (gc - chunk_base_of(p, n)) * kChunk;
  const int L = static_cast<int>(min(static_cast<long long>(kChunk), e - t0));

  Abort ab{p.err, &abort_s};
  if (tid == 0) {
    abort_s = 0;
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_init(&bar[2], 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc<128>(&tmem_base_s);

  // conv weights of this CTA's channels (q, k of key head kh; v of its G value heads)
  for (int x = tid; x < (2 + G) * 64; x += kPrepThreads) {
    const int pair = x % 64, grp = x / 64;  // grp 0 = q, 1 = k, 2.. = value head grp-2
    const long long ch0 = grp == 0 ? static_cast<long long>(kh) * kD
                        : grp == 1 ? static_cast<long long>(H_k + kh) * kD
                                   : static_cast<long long>(2 * H_k) * kD + static_cast<long long>(kh * G + grp - 2) * kD;
    sW[x] = __ldg(reinterpret_cast<const uint4*>(p.conv_w + (ch0 + 2 * pair) * kTaps));
  }
  __syncthreads();

  // identity rows 64..127 of the [P; I] image (hi = I, lo = 0)
  for (int x = tid; x < 64 * 8; x += kPrepThreads) {
    const int i = x >> 3, cc = x & 7;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (cc == (i >> 3)) {
      const int e8 = i & 7;
      w[e8 >> 1] = (e8 & 1) ? 0x3F800000u : 0x00003F80u;
    }
    *reinterpret_cast<uint4*>(sPI + sw128_off(64 + i, cc)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(sPI + 16384 + sw128_off(64 + i, cc)) = make_uint4(0u, 0u, 0u, 0u);
  }

  // ---- front end of q and k: token i, channels 32*qq .. 32*qq+31
  uint8_t* gQK = p.ws_qk + (gc * H_k + kh) * static_cast<long long>(kQKBytes);
  {
    const int i = tid >> 2, qq = tid & 3;
    const bool valid = i < L;
    for (int which = 0; which < 2; ++which) {
      const bf16* X = which ? p.k : p.q;
      const long long sx = which ? p.sk : p.sq;
      const long long chan0 = static_cast<long long>(which) * H_k * kD + static_cast<long long>(kh) * kD + 32 * qq;
      float y[32];
      if (valid) conv32(p, X + static_cast<long long>(kh) * kD + 32 * qq, sx, s, t0 + i, n, chan0, sW + which * 64 + 16 * qq, y);
      float ss = 0.f;
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        if (!valid) y[e2] = 0.f;
        ss = fmaf(y[e2], y[e2], ss);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      const float inv = rsqrtf(ss + 1e-6f) * (which == 0 ? p.scale : 1.0f);
      const int row = which * 64 + i, kb = qq >> 1;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float f[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) f[e2] = y[8 * c2 + e2] * inv;
        uint4 hi, lo;
        split8(f, hi, lo);
        const uint32_t off = kb * 16384u + sw128_off(row, (qq & 1) * 4 + c2);
        *reinterpret_cast<uint4*>(sQK + off) = hi;
        *reinterpret_cast<uint4*>(sQK + kQKImg + off) = lo;
        *reinterpret_cast<uint4*>(gQK + off) = hi;
        *reinterpret_cast<uint4*>(gQK + kQKImg + off) = lo;
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;

  // ---- [Q;K] K^T -> TMEM columns 0..63 (rows 0..63: Q K^T, rows 64..127: K K^T)
  if (tid == 0) {
    const uint32_t qh = smem_u32(sQK), ql = qh + kQKImg;
    const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t ko = (ks >> 2) * 16384u + (ks & 3) * 32u;
      umma_split(tbase, smem_desc(qh + ko, 16, 1024, Swz::k128), smem_desc(ql + ko, 16, 1024, Swz::k128),
                 smem_desc(qh + ko + 8192, 16, 1024, Swz::k128), smem_desc(ql + ko + 8192, 16, 1024, Swz::k128),
                 idesc, ks > 0);
    }
    umma_commit(&bar[0]);
  }

  // ---- gates of the key head's value heads (overlaps the MMA)
  for (int base = 0; base < G * 64; base += kPrepThreads) {
    const int x = base + tid;
    if (x < G * 64) {  // warp-uniform: G*64 is a multiple of 64
      const int j = x >> 6, i = x & 63, h = kh * G + j;
      const bool valid = i < L;
      float g = 0.f, beta = 0.f;
      if (valid) {
        const long long t = t0 + i;
        g = -expf(p.A_log[h]) * softplus_f(__bfloat162float(p.a[t * p.sa + h]));
        beta = sigmoid_f(__bfloat162float(p.b[t * p.sb + h]));
      }
      float v = g;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      sG[j * 64 + i] = v;
      sB[j * 64 + i] = beta;
    }
  }
  __syncthreads();
  for (int x = tid; x < G * 32; x += kPrepThreads) {
    const int j = x >> 5, i = 32 + (x & 31);
    sG[j * 64 + i] += sG[j * 64 + 31];
  }
  __syncthreads();
  // gate vectors for the scan: gamma_i, decay-to-end_i, gamma_C
  for (int x = tid; x < G * 256; x += kPrepThreads) {
    const int j = x >> 8, k2 = x & 255, h = kh * G + j;
    const float Glast = sG[j * 64 + (L - 1)];
    float val = 0.f;
    if (k2 < 64) val = expf(sG[j * 64 + k2]);
    else if (k2 < 128) val = (k2 - 64) < L ? expf(Glast - sG[j * 64 + (k2 - 64)]) : 0.f;
    else if (k2 == 128) val = expf(Glast);
    float* gdst = reinterpret_cast<float*>(p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes) + kPTBytes + kVBytes);
    gdst[k2] = val;
  }
  // ---- v_hat of the value heads (fp32): token i, channels 32*qq..+31
  {
    const int i = tid >> 2, qq = tid & 3;
    const bool valid = i < L;
    for (int j = 0; j < G; ++j) {
      const int h = kh * G + j;
      float y[32];
      if (valid) {
        conv32(p, p.v + static_cast<long long>(h) * kD + 32 * qq, p.sv, s, t0 + i, n,
               2LL * H_k * kD + static_cast<long long>(h) * kD + 32 * qq, sW + (2 + j) * 64 + 16 * qq, y);
      } else {
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) y[e2] = 0.f;
      }
      // [column block qq][quad q][token i] float4: a warp's reads of one quad are contiguous
      float4* dst = reinterpret_cast<float4*>(p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes) + kPTBytes) +
                    qq * 8 * 64 + i;
#pragma unroll
      for (int c2 = 0; c2 < 8; ++c2) dst[c2 * 64] = make_float4(y[4 * c2], y[4 * c2 + 1], y[4 * c2 + 2], y[4 * c2 + 3]);
    }
  }

  // ---- K K^T and Q K^T rows into registers: thread row = 32*(warp%4)+lane, columns cbase..cbase+31
  const int row = 32 * (warp & 3) + lane;
  const int cbase = 32 * (warp >> 2);
  const bool isQ = row < 64;
  const int ri = row & 63;
  float acc[32];
  if (mbar_wait_warp(&bar[0], 0, ab)) {
    tc_fence_after();
    tmem_ld32(tmem_addr(tbase, 32 * (warp & 3), cbase), acc);
    tmem_wait_ld();
  } else {
#pragma unroll
    for (int e2 = 0; e2 < 32; ++e2) acc[e2] = 0.f;
  }

  for (int j = 0; j < G; ++j) {
    const int h = kh * G + j;
    const float Gi = sG[j * 64 + ri];
    if (!isQ) {
      const float bi = sB[j * 64 + ri];
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        const int col = cbase + e2;
        sA[ri * kLdA + col] = col < ri ? bi * __expf(Gi - sG[j * 64 + col]) * acc[e2] : 0.f;
      }
    } else {
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float f[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const int col = cbase + 8 * c2 + e2;
          f[e2] = col <= ri ? __expf(Gi - sG[j * 64 + col]) * acc[8 * c2 + e2] : 0.f;
        }
        uint4 hi, lo;
        split8(f, hi, lo);
        *reinterpret_cast<uint4*>(sPI + sw128_off(ri, (cbase >> 3) + c2)) = hi;
        *reinterpret_cast<uint4*>(sPI + 16384 + sw128_off(ri, (cbase >> 3) + c2)) = lo;
      }
    }
    __syncthreads();
    solve_unit_lower(sA, sT, sM, tid);
    // T~ = T diag(beta): lower triangle incl. diagonal, as the MN-major B operand (row = k index)
    for (int x = tid; x < 64 * 8; x += kPrepThreads) {
      const int r = x >> 3, cc = x & 7;
      float f[8];
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        const int col = 8 * cc + e2;
        f[e2] = col <= r ? sT[r * kLdT + col] * sB[j * 64 + col] : 0.f;
      }
      uint4 hi, lo;
      split8(f, hi, lo);
      *reinterpret_cast<uint4*>(sTt + sw128_off(r, cc)) = hi;
      *reinterpret_cast<uint4*>(sTt + 8192 + sw128_off(r, cc)) = lo;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t pih = smem_u32(sPI), pil = pih + 16384, tth = smem_u32(sTt), ttl = tth + 8192;
      const uint32_t idesc = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_split(tbase + 64, smem_desc(pih + ks * 32, 16, 1024, Swz::k128),
                   smem_desc(pil + ks * 32, 16, 1024, Swz::k128), smem_desc(tth + ks * 2048, 8192, 1024, Swz::k128),
                   smem_desc(ttl + ks * 2048, 8192, 1024, Swz::k128), idesc, ks > 0);
      umma_commit(&bar[1]);
    }
    __syncwarp();
    float o[32];
    if (mbar_wait_warp(&bar[1], j & 1, ab)) {
      tc_fence_after();
      tmem_ld32(tmem_addr(tbase, 32 * (warp & 3), 64 + cbase), o);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) o[e2] = 0.f;
    }
    uint8_t* dst = p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes);
#pragma unroll
    for (int c2 = 0; c2 < 4; ++c2) {
      uint4 hi, lo;
      split8(o + 8 * c2, hi, lo);
      const uint32_t off = sw128_off(row, (cbase >> 3) + c2);
      *reinterpret_cast<uint4*>(dst + off) = hi;
      *reinterpret_cast<uint4*>(dst + kPTImg + off) = lo;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // drain: every MMA this CTA issued has completed before TMEM is released
  if (tid == 0) {
    umma_commit(&bar[2]);
    int drain_flag = 0;
    Abort drain{nullptr, &drain_flag};
    mbar_wait(&bar[2], 0, drain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc<128>(tbase);
}

// ============================================================ scan kernel

template <int DV>
struct ScanCfg {
  static constexpr int CS = 128 / DV;                  // CTAs per value head (cluster size)
  static constexpr int NB = DV / 32;                   // 32-column blocks per CTA
  static constexpr int TMEM_COLS = DV == 32 ? 256 : 512;
  static constexpr int COL_Z = 0;                      // S^T: lanes = d_k, DV columns
  // X = [Q;K] S^T and Y = [P T~; T~] R, each as two DV-column halves whose sum is
  // the product: (hi.hi + lo.hi | hi.lo) -- the hi and lo B operands sit side by
  // side along N so that A_hi [B_hi | B_lo] is one instruction.
  static constexpr int COL_X = DV;
  static constexpr int COL_Y = 3 * DV;
  // shared memory (offsets from a 1024-aligned base)
  static constexpr int OFF_GATE = kQKBytes;            // inside a [Q;K] stage
  static constexpr int QK_STAGE = kQKBytes + kGateBytes;
  static constexpr int OFF_PT = 2 * QK_STAGE;          // single [P T~; T~] buffer, hi then lo
  static constexpr int OFF_V = OFF_PT + kPTBytes;      // single v_hat slice, fp32 [DV/32][64][32]
  static constexpr int V_BYTES = 64 * DV * 4;
  static constexpr int OFF_OP = OFF_V + V_BYTES;       // S, R and U operands (hi image, then lo image)
  static constexpr int OP_IMG = 128 * DV * 2;
  static constexpr int OFF_NW = OFF_OP + 2 * OP_IMG;   // norm weight slice, fp32 [DV]
  static constexpr int OFF_SS = OFF_NW + 512;          // RMS partials [2][4][64] fp32
  static constexpr int SMEM = OFF_SS + 2048 + 1024;
  static constexpr uint32_t QK_TX = kQKBytes + kGateBytes;
};

// MN-major operand image with DV columns (8-element chunk index nch) and `krows` K-rows
template <int DV>
__device__ __forceinline__ uint32_t mn_off(uint32_t krow, uint32_t nch, uint32_t krows) {
  if constexpr (DV == 32) return sw64_off(krow, nch);
  else return (nch >> 3) * (krows * 128u) + sw128_off(krow, nch & 7u);
}

template <int DV>
__device__ __forceinline__ uint64_t mn_desc(uint32_t base, int ks, uint32_t krows) {
  if constexpr (DV == 32) return smem_desc(base + ks * 1024u, 512, 512, Swz::k64);
  else return smem_desc(base + ks * 2048u, krows * 128u, 1024, Swz::k128);
}

// [hi | lo] as one 2*DV-wide MN-major operand: the lo image is the next MN block, img_bytes on
template <int DV>
__device__ __forceinline__ uint64_t mn_desc_cat(uint32_t base_hi, int ks, uint32_t img_bytes) {
  if constexpr (DV == 32) return smem_desc(base_hi + ks * 1024u, img_bytes, 512, Swz::k64);
  else return smem_desc(base_hi + ks * 2048u, img_bytes, 1024, Swz::k128);
}

// write 32 fp32 values (one thread's row segment, columns 32*cc..) as hi/lo bf16 into an MN-major image
template <int DV>
__device__ __forceinline__ void store_split_row(uint8_t* img_hi, int img_bytes, uint32_t krow, int cc, uint32_t krows,
                                                const float* v) {
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint4 hi, lo;
    split8(v + 8 * q4, hi, lo);
    const uint32_t off = mn_off<DV>(krow, 4 * cc + q4, krows);
    *reinterpret_cast<uint4*>(img_hi + off) = hi;
    *reinterpret_cast<uint4*>(img_hi + img_bytes + off) = lo;
  }
}

template <int DV>
__global__ void __launch_bounds__(256, 1) scan_kernel(PrefillParams p) {
  using Cfg = ScanCfg<DV>;
  constexpr int CS = Cfg::CS, NB = Cfg::NB;
  if (p.cu && *p.ws_flag) return;  // same value in every CTA of a cluster
  extern __shared__ uint8_t scan_smem_raw[];
  uint8_t* sm = align1024(scan_smem_raw);
  __shared__ uint64_t qk_full[2], qk_empty[2], xyfree_b, mma2o_b, nfull_b[2], nack_b[2];
  __shared__ uint64_t pt_full, pt_empty, v_full, v_empty;
  __shared__ uint64_t mma1_b, mma2_b, mma3_b, drain_b, drain2_b;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = CS > 1 ? cluster_rank() : 0u;
  const int unit = blockIdx.x / CS;
  const int n_rank = unit / p.H_v, h = unit % p.H_v;
  const int n = (p.seq_order && p.N <= kMaxOrdered) ? p.seq_order[n_rank] : n_rank;
  const int G = p.H_v / p.H_k, kh = h / G;
  const int slice = static_cast<int>(rank);
  const long long s = seq_start(p, n), e = seq_start(p, n + 1);
  const int nc = static_cast<int>((e - s + kChunk - 1) / kChunk);
  const long long cb = chunk_base_of(p, n);

  Abort ab{p.err, &abort_s};
  float* sNW = reinterpret_cast<float*>(sm + Cfg::OFF_NW);
  float* sSS = reinterpret_cast<float*>(sm + Cfg::OFF_SS);
  uint8_t* sOP = sm + Cfg::OFF_OP;
  if (tid == 0) {
    abort_s = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(&qk_full[b], 1);
      mbar_init(&qk_empty[b], 1 + 64);
      if (CS > 1) {
        mbar_init(&nfull_b[b], (CS - 1) * 64);
        mbar_init(&nack_b[b], (CS - 1) * 64);
      }
    }
    mbar_init(&xyfree_b, 64);
    mbar_init(&mma2o_b, 1);
    mbar_init(&pt_full, 1);
    mbar_init(&pt_empty, 1);
    mbar_init(&v_full, 1);
    mbar_init(&v_empty, 64);
    mbar_init(&mma1_b, 1);
    mbar_init(&mma2_b, 1);
    mbar_init(&mma3_b, 1);
    mbar_init(&drain_b, 1);
    mbar_init(&drain2_b, 1);
    fence_mbar_init();
  }
  if (warp == 7) tmem_alloc<Cfg::TMEM_COLS>(&tmem_base_s);
  if (tid < DV) sNW[tid] = __bfloat162float(p.norm_w[slice * DV + tid]);
  tc_fence_before();
  __syncthreads();
  if (CS > 1) cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;
  const uint32_t op_hi = smem_u32(sOP), op_lo = op_hi + Cfg::OP_IMG;

  if (warp == 6) {
    // ------------------------------------------------ bulk-copy producer
    if (lane == 0) {
      int qk_issued[2] = {0, 0}, pt_issued = 0, v_issued = 0;
      for (int c = 0; c < nc; ++c) {
        const int st = c & 1;
        const long long gc = cb + c;
        const uint8_t* hb = p.ws_head + (gc * p.H_v + h) * static_cast<long long>(kHeadBytes);
        uint8_t* stage = sm + st * Cfg::QK_STAGE;
        if (c >= 2 && !mbar_wait(&qk_empty[st], ((c >> 1) - 1) & 1, ab, false, kBackoffNs)) break;
        mbar_arrive_expect_tx(&qk_full[st], Cfg::QK_TX);
        bulk_g2s(stage, p.ws_qk + (gc * p.H_k + kh) * static_cast<long long>(kQKBytes), kQKBytes, &qk_full[st]);
        bulk_g2s(stage + Cfg::OFF_GATE, hb + kPTBytes + kVBytes, kGateBytes, &qk_full[st]);
        ++qk_issued[st];
        if (c >= 1 && !mbar_wait(&pt_empty, (c - 1) & 1, ab, false, kBackoffNs)) break;
        mbar_arrive_expect_tx(&pt_full, kPTBytes);
        bulk_g2s(sm + Cfg::OFF_PT, hb, kPTBytes, &pt_full);
        ++pt_issued;
        if (c >= 1 && !mbar_wait(&v_empty, (c - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&v_full, Cfg::V_BYTES);
        bulk_g2s(sm + Cfg::OFF_V, hb + kPTBytes + slice * Cfg::V_BYTES, Cfg::V_BYTES, &v_full);
        ++v_issued;
      }
      // drain copies still in flight (only possible after an abort)
      int drain_flag = 0;
      Abort drain{nullptr, &drain_flag};
      for (int st = 0; st < 2; ++st)
        if (qk_issued[st] > 0) mbar_wait(&qk_full[st], (qk_issued[st] - 1) & 1, drain);
      if (pt_issued > 0) mbar_wait(&pt_full, (pt_issued - 1) & 1, drain);
      if (v_issued > 0) mbar_wait(&v_full, (v_issued - 1) & 1, drain);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------ state (threads 0..127), chain (64..127) and
    // the tensor-core issue: thread 0 issues X = [Q;K] S^T, thread 64 issues Y and the state
    // update.  Warps 0-3 pass the same three named barriers every chunk; each barrier ORs a
    // "something failed" predicate, so all four warps leave the loop at the same barrier.
    const int t = tid;  // TMEM lane = d_k index
    const uint32_t lb = 32 * warp;
    const long long srow0 = (static_cast<long long>(n) * p.H_v + h) * kD + static_cast<long long>(slice) * DV;
    const uint32_t idesc_1 = idesc_bf16(128, DV, false, true);       // A_lo B_hi
    const uint32_t idesc_2 = idesc_bf16(128, 2 * DV, false, true);   // A_hi [B_hi | B_lo]
    const uint32_t idesc_ku = idesc_bf16(128, DV, true, true);
    const uint32_t pt_hi = smem_u32(sm + Cfg::OFF_PT), pt_lo = pt_hi + kPTImg;
    const uint32_t dX = tbase + Cfg::COL_X, dY = tbase + Cfg::COL_Y;
    bool ok = true;
    for (int c = 0; c < nc; ++c) {
      const int st = c & 1;
      const float* gates = reinterpret_cast<const float*>(sm + st * Cfg::QK_STAGE + Cfg::OFF_GATE);
      const uint32_t qk_hi = smem_u32(sm + st * Cfg::QK_STAGE), qk_lo = qk_hi + kQKImg;
      // ---- state: S_{c-1} -> hi/lo operand image; S^T <- gamma_C S^T in TMEM
      bool w = c == 0 || mbar_wait_warp(&mma3_b, (c - 1) & 1, ab);
      if (w) w = mbar_wait_warp(&qk_full[st], (c >> 1) & 1, ab);
      if (w) {
        tc_fence_after();
        const float gC = gates[128];
        float v[NB][32];
        if (c == 0) {
#pragma unroll
          for (int cc = 0; cc < NB; ++cc)
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2)
              v[cc][e2] = p.state_in ? p.state_in[(srow0 + 32 * cc + e2) * kD + t] : 0.f;
        } else {
#pragma unroll
          for (int cc = 0; cc < NB; ++cc) tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Z + 32 * cc), v[cc]);
          tmem_wait_ld();  // one wait for all column blocks
        }
#pragma unroll
        for (int cc = 0; cc < NB; ++cc) {
          store_split_row<DV>(sOP, Cfg::OP_IMG, t, cc, 128, v[cc]);
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) v[cc][e2] *= gC;
          tmem_st32(tmem_addr(tbase, lb, Cfg::COL_Z + 32 * cc), v[cc]);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
      }
      tc_fence_before();
      if (bar_sync_or(1, 128, !w)) { ok = false; break; }
      bool issued = true;
      if (t == 0) {  // X = [Q;K] S^T
        issued = c == 0 || mbar_wait(&xyfree_b, (c - 1) & 1, ab);
        if (issued) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * 16384u + (ks & 3) * 32u;
            umma_bf16(dX, smem_desc(qk_hi + ko, 16, 1024, Swz::k128), mn_desc_cat<DV>(op_hi, ks, Cfg::OP_IMG),
                      idesc_2, ks > 0);
            umma_bf16(dX, smem_desc(qk_lo + ko, 16, 1024, Swz::k128), mn_desc<DV>(op_hi, ks, 128), idesc_1, true);
          }
          umma_commit(&mma1_b);
        }
      }
      // ---- chain: R = v_hat - gamma (K S^T)
      w = true;
      if (t >= 64) {
        const int i = t - 64;
        w = mbar_wait_warp(&mma1_b, c & 1, ab);
        if (w) w = mbar_wait_warp(&v_full, c & 1, ab);
        if (w) {
          tc_fence_after();
          const float gam = gates[i];
          const float4* vrow = reinterpret_cast<const float4*>(sm + Cfg::OFF_V);
#pragma unroll
          for (int cc = 0; cc < NB; ++cc) {
            float x[32], x2[32];
            tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_X + 32 * cc), x);
            tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_X + DV + 32 * cc), x2);
            tmem_wait_ld();
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) x[e2] += x2[e2];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 vv = vrow[(cc * 8 + q) * 64 + i];
              x[4 * q + 0] = fmaf(-gam, x[4 * q + 0], vv.x);
              x[4 * q + 1] = fmaf(-gam, x[4 * q + 1], vv.y);
              x[4 * q + 2] = fmaf(-gam, x[4 * q + 2], vv.z);
              x[4 * q + 3] = fmaf(-gam, x[4 * q + 3], vv.w);
            }
            store_split_row<DV>(sOP, Cfg::OP_IMG, i, cc, 64, x);
          }
          mbar_arrive(&v_empty);
          fence_proxy_async_smem();
        }
      }
      tc_fence_before();
      if (bar_sync_or(2, 128, !w || !issued)) { ok = false; break; }
      if (t == 64) {  // Y = [P T~; T~] R
        issued = mbar_wait(&pt_full, c & 1, ab);
        if (issued) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            umma_bf16(dY, smem_desc(pt_hi + ks * 32u, 16, 1024, Swz::k128), mn_desc_cat<DV>(op_hi, ks, Cfg::OP_IMG),
                      idesc_2, ks > 0);
            umma_bf16(dY, smem_desc(pt_lo + ks * 32u, 16, 1024, Swz::k128), mn_desc<DV>(op_hi, ks, 64), idesc_1, true);
          }
          umma_commit(&mma2_b);
          umma_commit(&mma2o_b);
          umma_commit(&pt_empty);
        }
      }
      // ---- chain: U_d = decay-to-end * U
      w = true;
      if (t >= 64) {
        const int i = t - 64;
        w = mbar_wait_warp(&mma2_b, c & 1, ab);
        if (w) {
          tc_fence_after();
          const float dcy = gates[64 + i];
#pragma unroll
          for (int cc = 0; cc < NB; ++cc) {
            float u[32], u2[32];
            tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Y + 32 * cc), u);
            tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Y + DV + 32 * cc), u2);
            tmem_wait_ld();
#pragma unroll
            for (int e2 = 0; e2 < 32; ++e2) u[e2] = (u[e2] + u2[e2]) * dcy;
            store_split_row<DV>(sOP, Cfg::OP_IMG, i, cc, 64, u);
          }
          fence_proxy_async_smem();
        }
      }
      tc_fence_before();
      if (bar_sync_or(3, 128, !w || !issued)) { ok = false; break; }
      if (t == 64) {  // S^T += K^T U_d
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          umma_split(tbase + Cfg::COL_Z, smem_desc(qk_hi + 8192u + ks * 2048u, 16384, 1024, Swz::k128),
                     smem_desc(qk_lo + 8192u + ks * 2048u, 16384, 1024, Swz::k128), mn_desc<DV>(op_hi, ks, 64),
                     mn_desc<DV>(op_lo, ks, 64), idesc_ku, true);
        umma_commit(&mma3_b);
        umma_commit(&qk_empty[st]);
      }
    }
    // every MMA this thread issued has completed before TMEM is read or released
    if (t == 0 || t == 64) {
      uint64_t* db = t == 0 ? &drain_b : &drain2_b;
      umma_commit(db);
      int drain_flag = 0;
      Abort drain{nullptr, &drain_flag};
      mbar_wait(db, 0, drain);
    }
    // final state of this slice
    if (p.state_out) {
      if (nc == 0) {
        for (int d = 0; d < DV; ++d)
          p.state_out[(srow0 + d) * kD + t] = p.state_in ? p.state_in[(srow0 + d) * kD + t] : 0.f;
      } else if (__all_sync(0xffffffffu, ok) && mbar_wait_warp(&mma3_b, (nc - 1) & 1, ab)) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < NB; ++cc) {
          float v[32];
          tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Z + 32 * cc), v);
          tmem_wait_ld();
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) p.state_out[(srow0 + 32 * cc + e2) * kD + t] = v[e2];
        }
      }
    }
  } else if (warp >= 4 && warp < 6) {
    // ------------------------------------------------ output (warps 4, 5): token i = TMEM lane i
    const int i = tid - 128;
    const uint32_t lb = 32 * (warp & 3);
    // z of the next chunk is loaded while this chunk's products are still running
    uint4 zbuf[NB * 4];
    auto load_z = [&](int c) {
      const long long tok = s + static_cast<long long>(c) * kChunk + i;
      const uint4* zrow = reinterpret_cast<const uint4*>(p.z + (tok < e ? tok : s) * p.sz +
                                                         static_cast<long long>(h) * kD + slice * DV);
#pragma unroll
      for (int q = 0; q < NB * 4; ++q) zbuf[q] = tok < e ? __ldg(zrow + q) : make_uint4(0u, 0u, 0u, 0u);
    };
    if (nc > 0) load_z(0);
    for (int c = 0; c < nc; ++c) {
      const int st = c & 1, pb = c & 1;
      if (!mbar_wait_warp(&qk_full[st], (c >> 1) & 1, ab, false, kBackoffNs)) break;
      const float gam = reinterpret_cast<const float*>(sm + st * Cfg::QK_STAGE + Cfg::OFF_GATE)[i];
      mbar_arrive(&qk_empty[st]);  // only gamma is read from the stage
      if (!mbar_wait_warp(&mma2o_b, c & 1, ab, false, kBackoffNs)) break;
      tc_fence_after();
      // o = gamma (X_a + X_b) + (Y_a + Y_b), kept in registers; per-32-column
      // partial sums of o^2 are combined in a fixed order for every slicing
      float o[DV];
      float part[NB];
#pragma unroll
      for (int cc = 0; cc < NB; ++cc) {
        float xa[32], xb2[32], ya[32], yb[32];
        tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_X + 32 * cc), xa);
        tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_X + DV + 32 * cc), xb2);
        tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Y + 32 * cc), ya);
        tmem_ld32(tmem_addr(tbase, lb, Cfg::COL_Y + DV + 32 * cc), yb);
        tmem_wait_ld();
        float ss = 0.f;
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) {
          const float v = fmaf(gam, xa[e2] + xb2[e2], ya[e2] + yb[e2]);
          o[32 * cc + e2] = v;
          ss = fmaf(v, v, ss);
        }
        part[cc] = ss;
      }
      tc_fence_before();
      mbar_arrive(&xyfree_b);  // X and Y may be overwritten by the next chunk's products
      float total;
      if constexpr (CS == 1) {
        total = part[0];
#pragma unroll
        for (int cc = 1; cc < NB; ++cc) total += part[cc];
      } else {
        if (c >= 2 && !mbar_wait_warp(&nack_b[pb], ((c >> 1) - 1) & 1, ab, true, kBackoffNs)) break;
#pragma unroll
        for (int cc = 0; cc < NB; ++cc) sSS[(pb * 4 + slice * NB + cc) * 64 + i] = part[cc];
        for (int r = 0; r < CS; ++r)
          if (r != slice) mbar_arrive_remote(&nfull_b[pb], static_cast<uint32_t>(r));
        if (!mbar_wait_warp(&nfull_b[pb], (c >> 1) & 1, ab, true, kBackoffNs)) break;
        float blk[4];
#pragma unroll
        for (int bidx = 0; bidx < 4; ++bidx) {
          const int owner = bidx / NB;
          blk[bidx] = owner == slice ? part[bidx % NB]
                                     : ld_shared_remote(sSS + (pb * 4 + bidx) * 64 + i, static_cast<uint32_t>(owner));
        }
        total = ((blk[0] + blk[1]) + blk[2]) + blk[3];
        for (int r = 0; r < CS; ++r)
          if (r != slice) mbar_arrive_remote(&nack_b[pb], static_cast<uint32_t>(r));
      }
      const float inv = rsqrtf(total * (1.0f / kD) + 1e-6f);
      const long long tok = s + static_cast<long long>(c) * kChunk + i;
      const bool valid = tok < e;
      uint4* orow = reinterpret_cast<uint4*>(p.out + ((valid ? tok : s) * p.H_v + h) * kD + slice * DV);
      uint4 ob[NB * 4];
#pragma unroll
      for (int q = 0; q < NB * 4; ++q) {
        float zz[8], f[8];
        unpack8(zbuf[q], zz);
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) f[e2] = o[8 * q + e2] * inv * sNW[8 * q + e2] * silu_fast(zz[e2]);
        ob[q] = pack8(f);
      }
      if (c + 1 < nc) load_z(c + 1);
      if (valid) {
#pragma unroll
        for (int q = 0; q < NB * 4; ++q) orow[q] = ob[q];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (CS > 1) cluster_sync_all();
  if (warp == 7) tmem_dealloc<Cfg::TMEM_COLS>(tbase);
}

template <int DV>
cudaError_t launch_scan(const PrefillParams& p, cudaStream_t stream) {
  using Cfg = ScanCfg<DV>;
  cudaError_t err = cudaFuncSetAttribute(scan_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.N) * p.H_v * Cfg::CS, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = Cfg::CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, scan_kernel<DV>, p);
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, int dv_slice, cudaStream_t stream, void* const* events) {
  cudaError_t err;
  if (p.cu) {
    setup_kernel<<<1, 1024, 0, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (p.conv_out) {
    const long long C_conv = static_cast<long long>(2 * p.H_k + p.H_v) * kD;
    conv_out_kernel<<<dim3(static_cast<unsigned>((C_conv + 255) / 256), p.N), 256, 0, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[0]), stream);
  if (p.n_chunks > 0) {
    const int smem = prep_smem_bytes(p.H_v / p.H_k);
    err = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    prep_kernel<<<dim3(static_cast<unsigned>(p.n_chunks), p.H_k), kPrepThreads, smem, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), stream);
  err = dv_slice == 32 ? launch_scan<32>(p, stream) : launch_scan<64>(p, stream);
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[2]), stream);
  return err;
}

}  // namespace gdn
