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
//   W = T diag(b gamma) K,   U0 = T diag(b) V,   U = U0 - W S^T,
//   O = diag(gamma) Q S^T + P U,   S <- gamma_C S + U^T diag(e^{G_C - G_j}) K.
//
// Two kernels (plus two small helpers):
//   prep (one CTA per chunk x key head, all chunks in parallel): conv + SiLU +
//     L2-norm front end of q and k, gates, [Q;K] K^T on tcgen05, the fp32 blocked
//     triangular solve, and per value head B_U = T diag(b), P, W = T diag(b gamma) K on
//     tcgen05 and v_hat = SiLU(conv(v)).  It writes the chunk's operand images to the
//     workspace.
//   scan (one CTA per sequence x value head): walks the chunks in order with
//     the whole fp32 state in tensor memory (lane = value row), the state and
//     U as bf16 hi/lo A operands read by tcgen05 straight from tensor memory.
//     Per chunk five tcgen05 products (V^T B_U^T, S W^T, S Q^T, U_d^T K,
//     U^T P^T) and the gated RMS-norm epilogue.
#define GDN_WAIT_OUT_OF_LINE  // the prefill kernels' waits share one polling loop (gdn_ptx.cuh)
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "../../include/gdn.h"
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

// Named barrier over `nthreads` threads that also ORs a per-thread predicate:
// every participant gets the same answer.
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
// [Q;K] operand image in shared memory: hi at +0, lo at +32768; K-block kb (channels
// 64 kb .. 64 kb + 63) at kb * 16384, rows 0..63 = Q tokens, rows 64..127 = K tokens.
// The K rows are the workspace's K image (four 8 KiB pieces, bulk-stored from here).
constexpr int kPrepOffQK = 0;
// Once the products that read Q have completed, the four 8 KiB Q pieces are scratch: per
// value head they stage P (hi, lo), then hold the B image B_W = T diag(beta gamma) (hi at 0,
// lo at 32768), then stage -W^T (lo rows 0..63, 64..127, hi rows 0..63, 64..127).
constexpr int kPrepOffBWhi = 0, kPrepOffBWlo = 32768;
// Region R (37 KiB) changes role through the kernel:
//   the raw q | k rows of the chunk (front-end input, rows of kRawStride bytes);
//   the identity B image of the q^T transpose;
//   per value head: T, A and the block-solve temp; then B_U = T diag(beta) (lo, hi) over
//   the dead A, staged for the workspace; then the staged (gamma Q)^T images (hi, lo).
constexpr int kPrepOffR = 65536;
constexpr int kRawStride = 2 * kD * 2 + 16;            // q row | k row, 16 B of padding against bank conflicts
constexpr int kPrepOffT = kPrepOffR;                   // T fp32                64*68*4
constexpr int kPrepOffA = kPrepOffT + 64 * kLdT * 4;   // A fp32                64*65*4
constexpr int kPrepOffM = kPrepOffA + 64 * kLdA * 4;   // block-solve temp      3*256*4
constexpr int kPrepRBytes = 64 * kLdT * 4 + 64 * kLdA * 4 + 3 * 256 * 4;
constexpr int kPrepOffG = kPrepOffR + kPrepRBytes;     // G cumsum   [8][64]
constexpr int kPrepOffB = kPrepOffG + 8 * 64 * 4;      // beta       [8][64]
constexpr int kPrepOffGam = kPrepOffB + 8 * 64 * 4;    // gamma = e^G [8][64]
constexpr int kPrepOffW = kPrepOffGam + 8 * 64 * 4;    // conv weights of the q and k channels, 2*128*8 B
constexpr int kPrepOffBU = kPrepOffA;                  // B_U lo | hi, once A is dead
constexpr int kVBatch = 3;                             // value heads whose raw v rows fit the [Q;K] region at once
static_assert((kChunk + kTaps - 1) * (kVBatch * kD * 2 + 16) <= 65536, "the staged v rows must fit the [Q;K] region");
constexpr int kPrepSmem = kPrepOffW + 2 * 128 * 8 + 1024;
static_assert((kChunk + kTaps - 1) * kRawStride <= kPrepRBytes, "the raw q | k rows must fit region R");
static_assert(kPrepOffBU % 1024 == 0 && 2 * kPImg <= 64 * kLdA * 4, "B_U must fit the A area");
static_assert(2 * kImg64 <= kPrepRBytes, "the (gamma Q)^T images must fit region R");
// tensor memory columns (256 per CTA, two CTAs per SM)
constexpr uint32_t kPrepColQK = 0;    // [Q;K] K^T: rows 0..63 Q K^T, rows 64..127 K K^T (64 columns)
constexpr uint32_t kPrepColQT = 64;   // q^T (lane = d_k, column = token)
constexpr uint32_t kPrepColW = 128;   // W^T (lane = d_k, column = token)

// W words of bf16 pairs from 2W fp32 values: hi[m] = (bf16(x[2m]), bf16(x[2m+1])) with
// the even element in the low half, lo[m] the same for the residuals x - hi.  One paired
// conversion per two values for each of hi and lo.
template <int W>
__device__ __forceinline__ void split_pairs(const float* x, uint32_t* hi, uint32_t* lo) {
#pragma unroll
  for (int m = 0; m < W; ++m) {
    const uint32_t h = pack_bf16x2(x[2 * m], x[2 * m + 1]);
    hi[m] = h;
    lo[m] = pack_bf16x2(x[2 * m] - bf16_lo(h), x[2 * m + 1] - bf16_hi(h));
  }
}

// The same split with the residual pair x - hi as one packed fp32x2 fma (hi * (-1) + x;
// exact, as x - hi is representable): fewer instructions, one more live register pair.
template <int W>
__device__ __forceinline__ void split_pairs_x2(const float* x, uint32_t* hi, uint32_t* lo) {
#pragma unroll
  for (int m = 0; m < W; ++m) {
    const uint32_t h = pack_bf16x2(x[2 * m], x[2 * m + 1]);
    hi[m] = h;
    const float2 r = __ffma2_rn(make_float2(bf16_lo(h), bf16_hi(h)), make_float2(-1.f, -1.f),
                                make_float2(x[2 * m], x[2 * m + 1]));
    lo[m] = pack_bf16x2(r.x, r.y);
  }
}

// hi = bf16(f), lo = bf16(f - hi) for 8 values, packed as 16-byte rows
__device__ __forceinline__ void split8(const float* f, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
  split_pairs<4>(f, h, l);
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// The 4-tap conv + SiLU of 32 channels from their raw inputs (tap j = token t - 3 + j, 4 x 8 bf16
// per tap): wsm holds the 32 channels' weights, 16 x uint4 (channels 2u, 2u+1; taps 0..3 each).
__device__ __forceinline__ void conv_taps(const uint4 (&xin)[kTaps][4], const uint4* wsm, float* y) {
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

// Conv (4 taps) + SiLU of 32 consecutive channels of one token.
//   src: the token-0 address of the group's first channel; rows before the sequence start
//   come from conv_in (or are zero).  w: the 32 channels' weights, 16 x uint4 (channels 2u,
//   2u+1; taps 0..3 each), in shared or global memory.  All 16 input loads are issued
//   before any arithmetic.
__device__ __forceinline__ void conv32(const PrefillParams& p, const bf16* src, long long src_stride,
                                       long long s, long long t, int n, long long conv_chan0, const uint4* w,
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
  conv_taps(xin, w, y);
}

// One block diagonal of the blocked inverse: for blocks (I, J = I - d),
//   M = sum_{K=J}^{I-1} A_IK T_KJ,   T_IJ = -T_II M
// with 16x16 blocks; each thread computes four adjacent columns of one row.
template <int d>
__device__ __forceinline__ void solve_level(const float* sA, float* sT, float* sM, int tid, int bar_id) {
  constexpr int nb = 4 - d;
  if (tid < nb * 64) {
    const int J = tid >> 6, I = J + d, ii = (tid >> 2) & 15, j4 = (tid & 3) * 4;
    const float* arow = sA + (16 * I + ii) * kLdA + 16 * J;
    const float* tcol = sT + (16 * J) * kLdT + 16 * J + j4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
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
  named_bar_sync(bar_id, kPrepThreads);
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
  named_bar_sync(bar_id, kPrepThreads);
}

// T = (I + A)^{-1} for a 64x64 strictly-lower A (fp32, shared memory), by 16x16
// blocks: diagonal blocks by forward substitution, then the three block
// diagonals below.  All 256 threads.
__device__ void solve_unit_lower(const float* sA, float* sT, float* sM, int tid, int bar_id) {
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
  named_bar_sync(bar_id, kPrepThreads);
  solve_level<1>(sA, sT, sM, tid, bar_id);
  solve_level<2>(sA, sT, sM, tid, bar_id);
  solve_level<3>(sA, sT, sM, tid, bar_id);
}

// D (+)= A B^T with both operands as hi/lo pairs: A_hi B_hi + A_hi B_lo + A_lo B_hi
__device__ __forceinline__ void umma_split(uint32_t d, uint64_t a_hi, uint64_t a_lo, uint64_t b_hi, uint64_t b_lo,
                                           uint32_t idesc, bool accumulate) {
  umma_bf16(d, a_hi, b_hi, idesc, accumulate);
  umma_bf16(d, a_hi, b_lo, idesc, true);
  umma_bf16(d, a_lo, b_hi, idesc, true);
}


// W words of bf16 pairs from 2W fp32 values: hi[m] = (bf16(x[2m]), bf16(x[2m+1])) with
// the even element in the low half, lo[m] the same for the residuals x - hi.
// Conv (4 taps) + SiLU of 32 consecutive channels of token i from the staged raw rows
// (row r holds token t0 - 3 + r; `off` = byte offset of the 32-channel group in a row).
__device__ __forceinline__ void conv32_rows(const uint8_t* raw, int i, int off, const uint4* wsm, float* y) {
  uint4 xin[kTaps][4];
#pragma unroll
  for (int j = 0; j < kTaps; ++j) {
    const uint4* row = reinterpret_cast<const uint4*>(raw + (i + j) * kRawStride + off);
#pragma unroll
    for (int g = 0; g < 4; ++g) xin[j][g] = row[g];
  }
  conv_taps(xin, wsm, y);
}

// Word of the gate area of (chunk gc, value head h) that the fused launch uses as the
// ready flag of the chunk's operands (the gate vectors occupy words 0 .. 128).
__device__ __forceinline__ int* ready_flag(const PrefillParams& p, long long gc, int h) {
  return reinterpret_cast<int*>(p.ws_head + (gc * p.H_v + h) * static_cast<long long>(kHeadBytes) + kHeadOffGate) +
         kReadyFlagWord;
}

// Prep of one (chunk gc, key head kh) by 256 threads: the CTA's threads 256 half .. 256 half + 255,
// shared memory at sm (1024-aligned), tensor-memory columns tbase .. tbase + 255 (allocated by
// the caller), mbarriers bar[4].  Block-wide steps use named barrier 2 + half over the 256 threads.
// `k` counts the items these threads ran before with the same mbarriers (initialised at k = 0;
// every wait takes its phase parity from k).  When go_flag is given, it is set once the first
// value head is done (or the item ends), which lets the other half of a CTA start out of phase.
// Writes the chunk's K image for the key head and, for each of its value heads, -W^T,
// (gamma Q)^T, P, B_U, v_hat and the gate vectors; the operand images leave shared memory as
// bulk stores (v_hat goes straight from registers).  In a fused launch it then publishes the chunk through the value heads' ready flags.
__device__ __forceinline__ void prep_body(const PrefillParams& p, long long gc, int kh, int half, uint8_t* sm,
                                          uint32_t tbase, uint64_t* bar, int* abort_s, int k, int* go_flag) {
  const int bar_id = 2 + half;
  uint8_t* sQK = sm + kPrepOffQK;
  uint8_t* sR = sm + kPrepOffR;
  float* sA = reinterpret_cast<float*>(sm + kPrepOffA);
  float* sT = reinterpret_cast<float*>(sm + kPrepOffT);
  float* sM = reinterpret_cast<float*>(sm + kPrepOffM);
  float* sG = reinterpret_cast<float*>(sm + kPrepOffG);
  float* sB = reinterpret_cast<float*>(sm + kPrepOffB);
  float* sGam = reinterpret_cast<float*>(sm + kPrepOffGam);
  uint4* sW = reinterpret_cast<uint4*>(sm + kPrepOffW);  // [2 * 64] channel pairs: q | k
  // bar: [Q;K] K^T, W (per head), drain, q^T

  const int tid = threadIdx.x & (kPrepThreads - 1), warp = tid >> 5, lane = tid & 31;
  const int H_k = p.H_k, H_v = p.H_v, G = H_v / H_k;
  const long long C_conv = static_cast<long long>(2 * H_k + H_v) * kD;

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
  const int nrows = L + kTaps - 1;  // raw rows of tokens t0 - 3 .. t0 + L - 1

  Abort ab{p.err, abort_s};
  const uint32_t ph = k & 1;  // phase parity of the once-per-item barriers
  if (tid == 0 && k == 0) {
    *abort_s = 0;
    for (int b = 0; b < 4; ++b) mbar_init(&bar[b], 1);
    fence_mbar_init();
  }
  named_bar_sync(bar_id, kPrepThreads);

  // ---- v_hat = SiLU(conv(v)) of the value heads, kVBatch heads at a time: their raw rows
  // (tokens t0 - 3 .. t0 + L - 1) are staged in the [Q;K] region with 16-byte asynchronous
  // copies (rows before the sequence start from conv_in, or zero), then each thread takes
  // 4 tokens x 8 channels of each head of the batch and stores the hi/lo pieces straight
  // into the workspace's MN-major image (rows past the chunk's end zero).  The raw q | k rows
  // of the front end are requested behind the first batch, so their latency overlaps it.
  for (int jb = 0; jb < G; jb += kVBatch) {
    const int nb = min(kVBatch, G - jb);
    const int vstride = nb * kD * 2 + 16;  // one staged row: nb heads x 128 channels, 16 B of padding
    for (int x = tid; x < nrows * nb * 16; x += kPrepThreads) {
      const int r = x / (nb * 16), piece = x % (nb * 16);
      const long long tau = t0 - (kTaps - 1) + r;
      const long long ch = static_cast<long long>(kh * G + jb) * kD + piece * 8;  // v channel
      uint8_t* dst = sQK + r * vstride + piece * 16;
      const bf16* src = nullptr;
      if (tau >= s) src = p.v + tau * p.sv + ch;
      else if (p.conv_in) src = p.conv_in + (static_cast<long long>(n) * 3 + 3 + (tau - s)) * C_conv + 2LL * H_k * kD + ch;
      if (src) cp_async16(dst, src);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    cp_async_commit();
    if (jb == 0) {
      // raw q | k rows into region R: 16-byte asynchronous copies by all threads (a warp moves
      // one 512-byte row per instruction); rows before the sequence start come from conv_in,
      // or are zero
      for (int x = tid; x < nrows * 32; x += kPrepThreads) {
        const int r = x >> 5, piece = x & 31, which = piece >> 4;
        const long long tau = t0 - (kTaps - 1) + r;
        uint8_t* dst = sR + r * kRawStride + piece * 16;
        const bf16* src = nullptr;
        if (tau >= s) src = (which ? p.k + tau * p.sk : p.q + tau * p.sq) + static_cast<long long>(kh) * kD;
        else if (p.conv_in)
          src = p.conv_in + (static_cast<long long>(n) * 3 + 3 + (tau - s)) * C_conv + static_cast<long long>(which * H_k + kh) * kD;
        if (src) cp_async16(dst, src + (piece & 15) * 8);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
      cp_async_commit();
      cp_async_wait_group<1>();  // the v rows (the q | k rows may still be in flight)
    } else {
      cp_async_wait_group<0>();
    }
    named_bar_sync(bar_id, kPrepThreads);
    const int cg = tid & 15, tg = tid >> 4;  // 8 channels, 4 tokens
    for (int jj = 0; jj < nb; ++jj) {
      const int h = kh * G + jb + jj;
      float2 wv[4][kTaps];
      {
        const uint4* wsrc = reinterpret_cast<const uint4*>(p.conv_w + (2LL * H_k * kD + static_cast<long long>(h) * kD + 8 * cg) * kTaps);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = __ldg(wsrc + q);
          wv[q][0] = make_float2(bf16_lo(w.x), bf16_lo(w.z));
          wv[q][1] = make_float2(bf16_hi(w.x), bf16_hi(w.z));
          wv[q][2] = make_float2(bf16_lo(w.y), bf16_lo(w.w));
          wv[q][3] = make_float2(bf16_hi(w.y), bf16_hi(w.w));
        }
      }
      const uint8_t* rsrc = sQK + jj * kD * 2 + cg * 16;
      uint8_t* gv = p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes) + kHeadOffV + (cg >> 3) * 8192;
      uint4 rw[4 + kTaps - 1];
#pragma unroll
      for (int r = 0; r < 4 + kTaps - 1; ++r) rw[r] = *reinterpret_cast<const uint4*>(rsrc + (4 * tg + r) * vstride);
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * tg + ii;
        float y[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // channel pair q: taps on rows ii .. ii + 3
          const uint32_t x0 = (&rw[ii].x)[q], x1 = (&rw[ii + 1].x)[q], x2 = (&rw[ii + 2].x)[q], x3 = (&rw[ii + 3].x)[q];
          float2 a = __fmul2_rn(wv[q][0], make_float2(bf16_lo(x0), bf16_hi(x0)));
          a = __ffma2_rn(wv[q][1], make_float2(bf16_lo(x1), bf16_hi(x1)), a);
          a = __ffma2_rn(wv[q][2], make_float2(bf16_lo(x2), bf16_hi(x2)), a);
          a = __ffma2_rn(wv[q][3], make_float2(bf16_lo(x3), bf16_hi(x3)), a);
          y[2 * q] = i < L ? silu_fast(a.x) : 0.f;
          y[2 * q + 1] = i < L ? silu_fast(a.y) : 0.f;
        }
        uint4 hi, lo;
        split8(y, hi, lo);
        const uint32_t off = sw128_off(i, cg & 7);
        if (ws_ok(p, gv + off, 16) && ws_ok(p, gv + kImg64 + off, 16)) {
          *reinterpret_cast<uint4*>(gv + off) = hi;
          *reinterpret_cast<uint4*>(gv + kImg64 + off) = lo;
        }
      }
    }
    named_bar_sync(bar_id, kPrepThreads);  // the staged rows are read: the region is free
  }

  // (raw q | k rows: requested above, behind the first v batch)

  // conv weights of this CTA's channels (q and k of key head kh)
  for (int x = tid; x < 2 * 64; x += kPrepThreads) {
    const int pair = x % 64, grp = x / 64;  // grp 0 = q, 1 = k
    const long long ch0 = static_cast<long long>(grp * H_k + kh) * kD;
    cp_async16(&sW[x], p.conv_w + (ch0 + 2 * pair) * kTaps);  // waited for with the raw rows
  }

  // ---- gates of the key head's value heads
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
  named_bar_sync(bar_id, kPrepThreads);
  for (int x = tid; x < G * 32; x += kPrepThreads) {
    const int j = x >> 5, i = 32 + (x & 31);
    sG[j * 64 + i] += sG[j * 64 + 31];
  }
  named_bar_sync(bar_id, kPrepThreads);
  for (int x = tid; x < G * 64; x += kPrepThreads) sGam[x] = expf(sG[x]);
  // ---- front end of q and k from the staged rows: token i, channels 32*qq .. 32*qq+31
  cp_async_wait_all();
  named_bar_sync(bar_id, kPrepThreads);
  {
    // a quarter-warp takes 8 consecutive tokens of one 32-channel group: the raw rows are
    // 528 bytes apart, so its 16-byte reads fall on 8 distinct bank groups
    const int i = (tid & 7) | ((tid >> 5) << 3), qq = (tid >> 3) & 3;
    const bool valid = i < L;
    for (int which = 0; which < 2; ++which) {
      float y[32];
      if (valid) conv32_rows(sR, i, which * kD * 2 + qq * 64, sW + which * 64 + 16 * qq, y);
      float ss = 0.f;
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        if (!valid) y[e2] = 0.f;
        ss = fmaf(y[e2], y[e2], ss);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 8);
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      const float inv = rsqrtf(ss + 1e-6f) * (which == 0 ? p.scale : 1.0f);
      const int row = which * 64 + i, kb = qq >> 1;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float f[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) f[e2] = y[8 * c2 + e2] * inv;
        uint4 hi, lo;
        split8(f, hi, lo);
        const uint32_t soff = kb * 16384u + sw128_off(row, (qq & 1) * 4 + c2);
        *reinterpret_cast<uint4*>(sQK + soff) = hi;
        *reinterpret_cast<uint4*>(sQK + 32768 + soff) = lo;
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  named_bar_sync(bar_id, kPrepThreads);
  tc_fence_after();

  // ---- the K image to the workspace (the K rows of the four K-block halves), and
  // [Q;K] K^T -> TMEM columns 0..63 (rows 0..63: Q K^T, rows 64..127: K K^T)
  if (tid == 0) {
    uint8_t* gK = p.ws_k + (gc * H_k + kh) * static_cast<long long>(kKBytes);
    if (ws_ok(p, gK, kKBytes)) {
#pragma unroll
      for (int piece = 0; piece < 4; ++piece)  // hi block 0, hi block 1, lo block 0, lo block 1
        bulk_s2g(gK + piece * 8192, sQK + piece * 16384 + 8192, 8192);
    }
    bulk_commit();
    const uint32_t qh = smem_u32(sQK), ql = qh + 32768;
    const uint32_t idesc = idesc_bf16(128, 64, false, false);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t ko = (ks >> 2) * 16384u + (ks & 3) * 32u;
      umma_split(tbase + kPrepColQK, smem_desc(qh + ko, 16, 1024, Swz::k128), smem_desc(ql + ko, 16, 1024, Swz::k128),
                 smem_desc(qh + ko + 8192, 16, 1024, Swz::k128), smem_desc(ql + ko + 8192, 16, 1024, Swz::k128),
                 idesc, ks > 0);
    }
    umma_commit(&bar[0]);
  }
  // gate vectors for the scan: gamma_i, decay-to-end_i (0 past the chunk's last token), gamma_C
  for (int x = tid; x < G * 256; x += kPrepThreads) {
    const int j = x >> 8, k2 = x & 255, h = kh * G + j;
    const float Glast = sG[j * 64 + (L - 1)];
    float val = 0.f;
    if (k2 < 64) {
      val = sGam[j * 64 + k2];
    } else if (k2 < 128) {
      val = (k2 - 64) < L ? expf(Glast - sG[j * 64 + (k2 - 64)]) : 0.f;
    } else if (k2 == 128) {
      val = expf(Glast);
    }
    float* gdst = reinterpret_cast<float*>(p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes) + kHeadOffGate);
    if (k2 != kReadyFlagWord && ws_ok(p, gdst + k2, 4)) gdst[k2] = val;
  }

  // identity B image for the q^T transpose, in region R (the raw rows are dead)
  for (int x = tid; x < 64 * 8; x += kPrepThreads) {
    const int i = x >> 3, cc = x & 7;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (cc == (i >> 3)) {
      const int e8 = i & 7;
      w[e8 >> 1] = (e8 & 1) ? 0x3F800000u : 0x00003F80u;  // bf16 1.0 in the element's half
    }
    *reinterpret_cast<uint4*>(sR + sw128_off(i, cc)) = make_uint4(w[0], w[1], w[2], w[3]);
  }

  // ---- K K^T and Q K^T rows into registers: thread row = 32*(warp%4)+lane, columns cbase..cbase+31
  const int row = 32 * (warp & 3) + lane;
  const int cbase = 32 * (warp >> 2);
  const bool isQ = row < 64;
  const int ri = row & 63;
  // (the [Q;K] K^T rows stay in tensor memory and are read again for each value head)
  const bool qk_ok = mbar_wait_warp(&bar[0], ph, ab);

  // ---- q^T (lane = d_k, column = token) into TMEM columns 64..127: Q_hi^T I + Q_lo^T I
  // with an identity B, exact in fp32
  fence_proxy_async_smem();
  tc_fence_before();
  named_bar_sync(bar_id, kPrepThreads);  // the identity is complete
  tc_fence_after();
  if (tid == 0) {
    const uint32_t qk = smem_u32(sQK), id = smem_u32(sR);
    const uint32_t idesc_t = idesc_bf16(128, 64, true, false);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t b = smem_desc(id + ks * 32u, 16, 1024, Swz::k128);
      umma_bf16(tbase + kPrepColQT, smem_desc(qk + ks * 2048u, 16384, 1024, Swz::k128), b, idesc_t, ks > 0);
      umma_bf16(tbase + kPrepColQT, smem_desc(qk + 32768u + ks * 2048u, 16384, 1024, Swz::k128), b, idesc_t, true);
    }
    umma_commit(&bar[3]);
  }
  __syncwarp();
  mbar_wait_warp(&bar[3], ph, ab);
  tc_fence_after();
  if (tid == 0) bulk_wait_read<0>();  // the K image has left shared memory
  named_bar_sync(bar_id, kPrepThreads);  // Q and the identity are dead: the Q pieces and region R are scratch

  for (int j = 0; j < G; ++j) {
    const int h = kh * G + j;
    uint8_t* hb = p.ws_head + (gc * H_v + h) * static_cast<long long>(kHeadBytes);
    const float Gi = sG[j * 64 + ri];
    float acc[32];
    if (qk_ok) {
      tmem_ld32(tmem_addr(tbase, 32 * (warp & 3), kPrepColQK + cbase), acc);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) acc[e2] = 0.f;
    }
    if (!isQ) {
      const float bi = sB[j * 64 + ri];
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        const int col = cbase + e2;
        sA[ri * kLdA + col] = col < ri ? bi * __expf(Gi - sG[j * 64 + col]) * acc[e2] : 0.f;
      }
    } else {
      // P_ij = e^{G_i - G_j} (q_i . k_j) for j <= i: K-major image (row i), staged hi in the Q
      // piece at 0 and lo in the one at 32768
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
        const uint32_t off = sw128_off(ri, (cbase >> 3) + c2);
        *reinterpret_cast<uint4*>(sQK + off) = hi;
        *reinterpret_cast<uint4*>(sQK + 32768 + off) = lo;
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(bar_id, kPrepThreads);
    if (tid == 0) {
      if (ws_ok(p, hb + kHeadOffP, 2 * kPImg)) {
        bulk_s2g(hb + kHeadOffP, sQK, kPImg);
        bulk_s2g(hb + kHeadOffP + kPImg, sQK + 32768, kPImg);
      }
      bulk_commit();
    }
    solve_unit_lower(sA, sT, sM, tid, bar_id);
    if (tid == 0) bulk_wait_read<0>();  // P has left the Q pieces
    named_bar_sync(bar_id, kPrepThreads);
    // B_W = T diag(beta gamma) into the Q pieces, B_U = T diag(beta) over the dead A: K-major
    // (row i, 64 j), lower triangle incl. diagonal
    uint8_t* sBU = sm + kPrepOffBU;  // lo | hi
    for (int x = tid; x < 64 * 8; x += kPrepThreads) {
      const int r = x >> 3, cc = x & 7;
      float fu[8], fw[8];
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        const int col = 8 * cc + e2;
        const float tb = col <= r ? sT[r * kLdT + col] * sB[j * 64 + col] : 0.f;
        fu[e2] = tb;
        fw[e2] = tb * sGam[j * 64 + col];
      }
      uint4 hi, lo;
      const uint32_t off = sw128_off(r, cc);
      split8(fw, hi, lo);
      *reinterpret_cast<uint4*>(sQK + kPrepOffBWhi + off) = hi;
      *reinterpret_cast<uint4*>(sQK + kPrepOffBWlo + off) = lo;
      split8(fu, hi, lo);
      *reinterpret_cast<uint4*>(sBU + off) = lo;
      *reinterpret_cast<uint4*>(sBU + kPImg + off) = hi;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(bar_id, kPrepThreads);
    tc_fence_after();
    if (tid == 0) {
      if (ws_ok(p, hb + kHeadOffBU, 2 * kPImg)) bulk_s2g(hb + kHeadOffBU, sBU, 2 * kPImg);
      bulk_commit();
      bulk_wait_read<0>();  // B_U has left region R before the product's completion frees it
      // W^T = K^T B_W^T: A = K (MN-major, rows = tokens), B = B_W (K-major)
      const uint32_t qk = smem_u32(sQK);
      const uint32_t idesc_w = idesc_bf16(128, 64, true, false);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        umma_split(tbase + kPrepColW, smem_desc(qk + 8192u + ks * 2048u, 16384, 1024, Swz::k128),
                   smem_desc(qk + 32768u + 8192u + ks * 2048u, 16384, 1024, Swz::k128),
                   smem_desc(qk + kPrepOffBWhi + ks * 32u, 16, 1024, Swz::k128),
                   smem_desc(qk + kPrepOffBWlo + ks * 32u, 16, 1024, Swz::k128), idesc_w, ks > 0);
      umma_commit(&bar[1]);
    }
    __syncwarp();
    if (mbar_wait_warp(&bar[1], (k * G + j) & 1, ab)) {
      tc_fence_after();
      // -W^T row d_k = 32 (warp % 4) + lane, tokens 32 (warp / 4) .. +31: staged lo rows
      // 0..63 | 64..127 in the Q pieces at 0 | 16384, hi rows 0..63 | 64..127 at 32768 | 49152
      const int kr = 32 * (warp & 3) + lane, half = warp >> 2;
      float o[32];
      tmem_ld32(tmem_addr(tbase, 32 * (warp & 3), kPrepColW + 32 * half), o);
      tmem_wait_ld();
      const uint32_t half_off = kr < 64 ? 0u : 16384u;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float f[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) f[e2] = -o[8 * c2 + e2];
        uint4 hi, lo;
        split8(f, hi, lo);
        const uint32_t off = sw128_off(kr & 63, 4 * half + c2);
        *reinterpret_cast<uint4*>(sQK + half_off + off) = lo;
        *reinterpret_cast<uint4*>(sQK + 32768 + half_off + off) = hi;
      }
      // (gamma Q)^T row d_k = kr, the same 32 tokens: staged in region R, hi rows 0..63 | 64..127
      // then lo rows 0..63 | 64..127
      tmem_ld32(tmem_addr(tbase, 32 * (warp & 3), kPrepColQT + 32 * half), o);
      tmem_wait_ld();
      const uint32_t rhalf = kr < 64 ? 0u : 8192u;
#pragma unroll
      for (int c2 = 0; c2 < 4; ++c2) {
        float f[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) f[e2] = o[8 * c2 + e2] * sGam[j * 64 + 32 * half + 8 * c2 + e2];
        uint4 hi, lo;
        split8(f, hi, lo);
        const uint32_t off = rhalf + sw128_off(kr & 63, 4 * half + c2);
        *reinterpret_cast<uint4*>(sR + off) = hi;
        *reinterpret_cast<uint4*>(sR + kImg64 + off) = lo;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_bar_sync(bar_id, kPrepThreads);
    tc_fence_after();
    if (tid == 0) {
      uint8_t* wd = hb + kHeadOffW;  // -W^T lo | -W^T hi | (gamma Q)^T hi | (gamma Q)^T lo
      if (ws_ok(p, wd, 2 * kWBytes)) {
        bulk_s2g(wd, sQK, 8192);
        bulk_s2g(wd + 8192, sQK + 16384, 8192);
        bulk_s2g(wd + 16384, sQK + 32768, 8192);
        bulk_s2g(wd + 24576, sQK + 49152, 8192);
        bulk_s2g(hb + kHeadOffGQ, sR, 2 * kImg64);
      }
      bulk_commit();
      bulk_wait_read<0>();  // the staging areas (Q pieces, region R) are rewritten by the next value head
    }
    named_bar_sync(bar_id, kPrepThreads);
    if (go_flag && tid == 0) *reinterpret_cast<volatile int*>(go_flag) = 1;
  }
  if (go_flag && tid == 0) *reinterpret_cast<volatile int*>(go_flag) = 1;

  // drain: every MMA this CTA issued and every bulk store has completed
  if (tid == 0) {
    umma_commit(&bar[2]);
    int drain_flag = 0;
    Abort drain{nullptr, &drain_flag};
    mbar_wait(&bar[2], ph, drain);
    bulk_wait<0>();
  }
  if (p.fused_scan_ctas > 0) {
    // publish: every store of this chunk (bulk images drained above, v_hat and gate vectors
    // by all threads) is visible before the value heads' ready flags
    __threadfence();
    named_bar_sync(bar_id, kPrepThreads);
    if (tid == 0) {
      fence_proxy_async_global();
      __threadfence();
      for (int j = 0; j < G; ++j) st_release_gpu(ready_flag(p, gc, kh * G + j), 1);
    }
  }
  tc_fence_before();
  named_bar_sync(bar_id, kPrepThreads);
}


__global__ void __launch_bounds__(kPrepThreads, 2) prep_kernel(PrefillParams p) {
  if (p.cu && *p.ws_flag) return;
  extern __shared__ uint8_t prep_smem_raw[];
  __shared__ uint64_t bar[4];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  if (threadIdx.x < 32) tmem_alloc<256>(&tmem_base_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;
  prep_body(p, blockIdx.x, blockIdx.y, 0, align1024(prep_smem_raw), tbase, bar, &abort_s, 0, nullptr);
  if (threadIdx.x < 32) tmem_dealloc<256>(tbase);  // prep_body ends with a barrier after its last use
}

// ============================================================ scan kernel
//
// One CTA per (sequence, value head); the whole 128 x 128 state lives in tensor
// memory with lane = d_v row.  Per chunk, every product summed over the hi/lo
// split terms (hi.hi + hi.lo + lo.hi):
//   [U^T | O^T]  = V^T [B_U^T | 0] + S [-W^T | (gamma Q)^T]   (U0 from shared-memory operands
//                  first, off the chain; then the U half, committed on its own so that the U
//                  conversion starts early, then the O half behind it)
//   S   = gamma_C S + (U^T diag(e^{G_C - G_j})) K   (A = U_d hi/lo from TMEM)
//   O^T += U^T P^T                      (A = U hi/lo from TMEM)
//   then the gated RMS-norm of o_i over d_v.
// Warps 0-7 (thread = d_v row; warps w and w + 4 share a TMEM lane quarter and
// split its columns) convert S and U between fp32 accumulators and bf16 hi/lo
// operands in tensor memory, each conversion publishing first the part the next
// product waits for; warps 8-11 run the output stage (the first product of o overwrites
// O once they have read it); warp 12 lane 0 issues the MMAs; warp 13 lane 0 issues the bulk copies
// (v_hat, B_U, W | gamma Q, K, P single-buffered, gates double-buffered).

constexpr int kScanThreads = 448;
constexpr int kScanBar = 15;  // named barrier of the scan's CTA-wide steps
constexpr int kWarpIssue = 12, kWarpProd = 13;
// tensor memory columns (512 allocated)
constexpr uint32_t kColS = 0;      // S fp32, 128 columns (d_k)
constexpr uint32_t kColSH = 128;   // S hi, bf16 pairs along d_k (64 columns)
constexpr uint32_t kColSL = 192;   // S lo
// [U2 | U1 | O1 | O2], 4 x 64 columns:
//   U2 = V_hi B_U_lo - S_hi W_lo,  U1 = V_hi B_U_hi + V_lo B_U_hi - S_hi W_hi - S_lo W_hi,
//   O1 = S_hi gQ_hi + S_lo gQ_hi + U_hi P_hi + U_lo P_hi,  O2 = S_hi gQ_lo + U_hi P_lo
//   (O1 | O2 start from the first K step of S_hi gQ, without accumulation)
constexpr uint32_t kColU2 = 256;   //   U^T = U2 + U1
constexpr uint32_t kColU1 = 320;
constexpr uint32_t kColO = 384;    //   o = O1 + O2
// After the U conversion, in place: the chain warp of token half th (tokens 32 th .. +31)
// read U2 / U1 columns 256 + 32 th / 320 + 32 th and writes there, 16 columns each,
//   U hi at 256 + 32 th, U lo at 272 + 32 th, U_d hi at 320 + 32 th, U_d lo at 336 + 32 th,
// so K step ks (tokens 16 ks .. +15) of an A operand sits at base + 32 (ks / 2) + 8 (ks % 2).
constexpr uint32_t kColUH = 256;
constexpr uint32_t kColUL = 272;
constexpr uint32_t kColUDH = 320;
constexpr uint32_t kColUDL = 336;
__host__ __device__ constexpr uint32_t ucol(uint32_t base, int ks) { return base + 32u * (ks >> 1) + 8u * (ks & 1); }
// shared memory (offsets from a 1024-aligned base)
constexpr int kScOffW = 0;                             // -W^T lo | -W^T hi | (gQ)^T hi | (gQ)^T lo
constexpr int kScOffK = kScOffW + 2 * kWBytes;         // K hi | K lo
constexpr int kScOffP = kScOffK + 2 * kImg64;          // P hi | P lo
constexpr int kScOffBU = kScOffP + 2 * kPImg;          // B_U lo | B_U hi
constexpr int kScOffV = kScOffBU + 2 * kPImg;          // v_hat hi | lo (MN-major: row = token, two 64-channel blocks)
constexpr int kScOffO = kScOffV + 2 * kImg64;          // o fp32 [64 tokens][128 d_v] for the token-major epilogue
constexpr int kScOffG = kScOffO + 64 * kD * 4;         // 2 stages of gates
constexpr int kScSmem = kScOffG + 2 * kGateBytes + 1024;

// The scan of one (sequence, value head) (`blk` = sequence rank * H_v + value head) by the
// CTA's first 448 threads (kIssueUnroll: unrolling of the MMA issue loops), with shared memory at sm (1024-aligned, kScSmem - 1024 bytes).
// CTA-wide steps use named barrier kScanBar.
template <int kIssueUnroll>
__device__ __forceinline__ void scan_body(const PrefillParams& p, int blk, uint8_t* sm) {
  __shared__ uint64_t g_full[2], g_free[2];
  __shared__ uint64_t w_full, w_free, k_full, k_free, p_full, p_free, bu_full, bu_free;
  __shared__ uint64_t v_full, v_free;
  __shared__ uint64_t s_conv, u_conv, u_conv2, u_done, s_done, y_done, o_free, drain_b;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_rank = blk / p.H_v, h = blk % p.H_v;
  const int n = (p.seq_order && p.N <= kMaxOrdered) ? p.seq_order[n_rank] : n_rank;
  const int G = p.H_v / p.H_k, kh = h / G;
  const long long s = seq_start(p, n), e = seq_start(p, n + 1);
  const int nc = static_cast<int>((e - s + kChunk - 1) / kChunk);
  const long long cb = chunk_base_of(p, n);

  Abort ab{p.err, &abort_s};
  if (tid == 0) {
    abort_s = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(&g_full[b], 1);
      mbar_init(&g_free[b], 256);
    }
    mbar_init(&w_full, 1);
    mbar_init(&w_free, 1);
    mbar_init(&k_full, 1);
    mbar_init(&k_free, 1);
    mbar_init(&p_full, 1);
    mbar_init(&p_free, 1);
    mbar_init(&bu_full, 1);
    mbar_init(&bu_free, 1);
    mbar_init(&v_full, 1);
    mbar_init(&v_free, 1);
    mbar_init(&s_conv, 256);
    mbar_init(&u_conv, 256);
    mbar_init(&u_conv2, 256);
    mbar_init(&u_done, 1);
    mbar_init(&s_done, 1);
    mbar_init(&y_done, 1);
    mbar_init(&o_free, 128);
    mbar_init(&drain_b, 1);
    fence_mbar_init();
  }
  if (warp == kWarpIssue) tmem_alloc<512>(&tmem_base_s);
  tc_fence_before();
  named_bar_sync(kScanBar, kScanThreads);
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;

  if (warp < 8) {
    // ------------------------------------------------ S and U conversions; thread = d_v row v,
    // columns / tokens of half th
    const int v = 32 * (warp & 3) + lane, th = warp >> 2;
    const uint32_t tl = tmem_addr(tbase, 32 * (warp & 3), 0);
    const long long srow = ((static_cast<long long>(n) * p.H_v + h) * kD + v) * kD;
    bool ok = true;
    for (int c = 0; c < nc && ok; ++c) {
      const int gs = c & 1;
      const float* gates = reinterpret_cast<const float*>(sm + kScOffG + gs * kGateBytes);
      // ---- S_c (columns 64 th .. +63) -> hi/lo operand; then S <- gamma_C S for the update
      ok = c == 0 || mbar_wait_warp(&s_done, (c - 1) & 1, ab);
      if (ok) ok = mbar_wait_warp(&g_full[gs], (c >> 1) & 1, ab);
      if (!ok) break;
      tc_fence_after();
      float sv[64];
      if (c == 0) {
        if (p.state_in) {
          const float4* src = reinterpret_cast<const float4*>(p.state_in + srow + 64 * th);
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 f = __ldg(src + q4);
            sv[4 * q4] = f.x; sv[4 * q4 + 1] = f.y; sv[4 * q4 + 2] = f.z; sv[4 * q4 + 3] = f.w;
          }
        } else {
#pragma unroll
          for (int e2 = 0; e2 < 64; ++e2) sv[e2] = 0.f;
        }
      } else {
        tmem_ld32(tl + kColS + 64 * th, sv);
        tmem_ld32(tl + kColS + 64 * th + 32, sv + 32);
        tmem_wait_ld();
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t hi[16], lo[16];
        split_pairs_x2<16>(sv + 32 * cc, hi, lo);
        tmem_st16(tl + kColSH + 32 * th + 16 * cc, hi);
        tmem_st16(tl + kColSL + 32 * th + 16 * cc, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&s_conv);
      const float gC = gates[128];
#pragma unroll
      for (int e2 = 0; e2 < 64; e2 += 2) {
        const float2 r = __fmul2_rn(make_float2(sv[e2], sv[e2 + 1]), make_float2(gC, gC));
        sv[e2] = r.x;
        sv[e2 + 1] = r.y;
      }
      tmem_st32(tl + kColS + 64 * th, sv);
      tmem_st32(tl + kColS + 64 * th + 32, sv + 32);
      // ---- U^T = U2 + U1 for tokens 32 th .. +31: U_d = U^T diag(decay-to-end) first (the
      // state update waits for it), then U (the output product waits for it)
      ok = mbar_wait_warp(&u_done, c & 1, ab);
      if (!ok) break;
      tc_fence_after();
      float u[32], ud[32];
      {
        float u1[32];
        tmem_ld32(tl + kColU2 + 32 * th, u);
        tmem_ld32(tl + kColU1 + 32 * th, u1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 r = __fadd2_rn(make_float2(u1[i], u1[i + 1]), make_float2(u[i], u[i + 1]));
          u[i] = r.x;
          u[i + 1] = r.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 d = *reinterpret_cast<const float2*>(gates + 64 + 32 * th + i);
        const float2 r = __fmul2_rn(make_float2(u[i], u[i + 1]), d);
        ud[i] = r.x;
        ud[i + 1] = r.y;
      }
      mbar_arrive(&g_free[gs]);  // the chunk's gates have been read for the last time
      {
        uint32_t hi[16], lo[16];
        split_pairs_x2<16>(ud, hi, lo);
        tmem_st16(tl + kColUDH + 32 * th, hi);
        tmem_st16(tl + kColUDL + 32 * th, lo);
      }
      tmem_wait_st();  // also covers the rescaled S
      tc_fence_before();
      mbar_arrive(&u_conv);
      {
        uint32_t hi[16], lo[16];
        split_pairs_x2<16>(u, hi, lo);
        tmem_st16(tl + kColUH + 32 * th, hi);
        tmem_st16(tl + kColUL + 32 * th, lo);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&u_conv2);
    }
    // final state of this head (row v, columns 64 th .. +63)
    if (p.state_out) {
      if (nc == 0) {
        for (int k = 64 * th; k < 64 * th + 64; ++k) p.state_out[srow + k] = p.state_in ? p.state_in[srow + k] : 0.f;
      } else if (__all_sync(0xffffffffu, ok) && mbar_wait_warp(&s_done, (nc - 1) & 1, ab)) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float sv2[32];
          tmem_ld32(tl + kColS + 64 * th + 32 * cc, sv2);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(p.state_out + srow + 64 * th + 32 * cc);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) dst[q4] = make_float4(sv2[4 * q4], sv2[4 * q4 + 1], sv2[4 * q4 + 2], sv2[4 * q4 + 3]);
        }
      }
    }
  } else if (warp == kWarpIssue) {
    // ------------------------------------------------ tensor-core issue (one thread)
    if (lane == 0) {
      const uint32_t idesc_v = idesc_bf16(128, 128, true, false);   // v_hi^T [B_U lo | B_U hi] (A MN-major)
      const uint32_t idesc_v2 = idesc_bf16(128, 64, true, false);   // v_lo^T B_U hi
      const uint32_t idesc_u = idesc_bf16(128, 128, false, true);   // S_hi [-W_lo | -W_hi], S_hi [gQ_hi | gQ_lo] (B MN-major)
      const uint32_t idesc_u2 = idesc_bf16(128, 64, false, true);   // S_lo (-W_hi), S_lo gQ_hi
      const uint32_t idesc_s = idesc_bf16(128, 128, false, true);   // U_d K (K MN-major, N = d_k)
      const uint32_t idesc_y = idesc_bf16(128, 128, false, false);  // U_hi [P_hi | P_lo] (K-major)
      const uint32_t idesc_y2 = idesc_bf16(128, 64, false, false);  // U_lo P_hi
      const uint32_t wq = smem_u32(sm + kScOffW);
      const uint32_t k_hi = smem_u32(sm + kScOffK), k_lo = k_hi + kImg64;
      const uint32_t p_hi = smem_u32(sm + kScOffP);
      const uint32_t bu_lo = smem_u32(sm + kScOffBU), bu_hi = bu_lo + kPImg;
      const uint32_t v_hi = smem_u32(sm + kScOffV), v_lo = v_hi + kImg64;
      for (int c = 0; c < nc; ++c) {
        // U0 = v_hat^T B_U^T into [U2 | U1], once the previous chunk's update and output
        // products (their commit covers every earlier MMA) have read the U columns
        if (c > 0 && !mbar_wait(&y_done, (c - 1) & 1, ab)) break;
        if (!mbar_wait(&v_full, c & 1, ab)) break;
        if (!mbar_wait(&bu_full, c & 1, ab)) break;
        tc_fence_after();
#pragma unroll kIssueUnroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ah = smem_desc(v_hi + ks * 2048u, 8192, 1024, Swz::k128);
          const uint64_t al = smem_desc(v_lo + ks * 2048u, 8192, 1024, Swz::k128);
          const uint64_t b2 = smem_desc(bu_lo + ks * 32u, 16, 1024, Swz::k128);  // 128 rows: B_U lo then hi
          const uint64_t bh = smem_desc(bu_hi + ks * 32u, 16, 1024, Swz::k128);
          umma_bf16(tbase + kColU2, ah, b2, idesc_v, ks > 0);
          umma_bf16(tbase + kColU1, al, bh, idesc_v2, true);
        }
        umma_commit(&v_free);
        umma_commit(&bu_free);
        // the chain's product onto U0: [U2 | U1] += S_hi [-W_lo | -W_hi], U1 += S_lo (-W_hi); its
        // commit lets the U conversion start while the state's part of o is issued and runs
        // behind it, [O1 | O2] = S_hi [gQ_hi | gQ_lo], O1 += S_lo gQ_hi, once the output warps
        // have read the previous chunk's O (the first product overwrites it)
        if (!mbar_wait(&s_conv, c & 1, ab)) break;
        if (!mbar_wait(&w_full, c & 1, ab)) break;
        tc_fence_after();
#pragma unroll kIssueUnroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bw = smem_desc(wq + ks * 2048u, kImg64, 1024, Swz::k128);
          const uint64_t bw2 = smem_desc(wq + kImg64 + ks * 2048u, kImg64, 1024, Swz::k128);
          umma_bf16_ts(tbase + kColU2, tbase + kColSH + 8 * ks, bw, idesc_u, true);
          umma_bf16_ts(tbase + kColU1, tbase + kColSL + 8 * ks, bw2, idesc_u2, true);
        }
        umma_commit(&u_done);
        if (!mbar_wait(&o_free, c & 1, ab)) break;
        tc_fence_after();
#pragma unroll kIssueUnroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t bq = smem_desc(wq + 2 * kImg64 + ks * 2048u, kImg64, 1024, Swz::k128);
          umma_bf16_ts(tbase + kColO, tbase + kColSH + 8 * ks, bq, idesc_u, ks > 0);
          umma_bf16_ts(tbase + kColO, tbase + kColSL + 8 * ks, bq, idesc_u2, true);
        }
        umma_commit(&w_free);
        if (!mbar_wait(&u_conv, c & 1, ab)) break;
        if (!mbar_wait(&k_full, c & 1, ab)) break;
        tc_fence_after();
        // S += U_d^T K (onto gamma_C S)
#pragma unroll kIssueUnroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bh = smem_desc(k_hi + ks * 2048u, 8192, 1024, Swz::k128);
          const uint64_t bl = smem_desc(k_lo + ks * 2048u, 8192, 1024, Swz::k128);
          umma_bf16_ts(tbase + kColS, tbase + ucol(kColUDH, ks), bh, idesc_s, true);
          umma_bf16_ts(tbase + kColS, tbase + ucol(kColUDH, ks), bl, idesc_s, true);
          umma_bf16_ts(tbase + kColS, tbase + ucol(kColUDL, ks), bh, idesc_s, true);
        }
        umma_commit(&s_done);
        umma_commit(&k_free);
        if (!mbar_wait(&u_conv2, c & 1, ab)) break;
        if (!mbar_wait(&p_full, c & 1, ab)) break;
        tc_fence_after();
        // [O1 | O2] += U_hi [P_hi | P_lo], O1 += U_lo P_hi
#pragma unroll kIssueUnroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t b2 = smem_desc(p_hi + ks * 32u, 16, 1024, Swz::k128);  // 128 rows: P hi then P lo
          umma_bf16_ts(tbase + kColO, tbase + ucol(kColUH, ks), b2, idesc_y, true);
          umma_bf16_ts(tbase + kColO, tbase + ucol(kColUL, ks), b2, idesc_y2, true);
        }
        umma_commit(&y_done);
        umma_commit(&p_free);
      }
      // every MMA issued has completed before TMEM is read for the last time or released
      umma_commit(&drain_b);
      int drain_flag = 0;
      Abort drain{nullptr, &drain_flag};
      mbar_wait(&drain_b, 0, drain);
    }
    __syncwarp();
  } else if (warp == kWarpProd) {
    // ------------------------------------------------ bulk-copy producer (lane 0)
    if (lane == 0) {
      // Order of need: v_hat, B_U, W | gamma Q, K, P of chunk c (single stages, each refilled as
      // soon as the product that reads it has completed), then the double-buffered gates of
      // chunk c + 1.
      int n_g[2] = {0, 0}, n_v = 0, n_bu = 0, n_w = 0, n_k = 0, n_p = 0;
      // a bulk load into shared memory with its byte count on `bar`; one outside the workspace
      // (debug build) is skipped and the barrier completes without data
      auto load = [&](void* dst, const uint8_t* src, uint32_t bytes, uint64_t* bar) {
        if (ws_ok(p, src, bytes)) {
          mbar_arrive_expect_tx(bar, bytes);
          bulk_g2s(dst, src, bytes, bar);
        } else {
          mbar_arrive(bar);
        }
      };
      auto head_blob = [&](int c) {
        return p.ws_head + ((cb + c) * p.H_v + h) * static_cast<long long>(kHeadBytes);
      };
      auto load_gates = [&](int c) -> bool {  // chunk c into stage c & 1
        const int st = c & 1;
        // fused launch: chunk c's operands (read from here on) are published by its prep
        if (p.fused_scan_ctas > 0 && !flag_wait(ready_flag(p, cb + c, h), ab, kBackoffNs)) return false;
        if (c >= 2 && !mbar_wait(&g_free[st], ((c >> 1) - 1) & 1, ab, false, kBackoffNs)) return false;
        load(sm + kScOffG + st * kGateBytes, head_blob(c) + kHeadOffGate, kGateBytes, &g_full[st]);
        ++n_g[st];
        return true;
      };
      bool ok = nc == 0 || load_gates(0);
      for (int c = 0; c < nc && ok; ++c) {
        const uint8_t* hb = head_blob(c);
        const uint8_t* kb = p.ws_k + ((cb + c) * p.H_k + kh) * static_cast<long long>(kKBytes);
        if (c >= 1 && !mbar_wait(&v_free, (c - 1) & 1, ab, false, kBackoffNs)) break;
        load(sm + kScOffV, hb + kHeadOffV, 2 * kImg64, &v_full);
        ++n_v;
        if (c >= 1 && !mbar_wait(&bu_free, (c - 1) & 1, ab, false, kBackoffNs)) break;
        load(sm + kScOffBU, hb + kHeadOffBU, 2 * kPImg, &bu_full);
        ++n_bu;
        if (c >= 1 && !mbar_wait(&w_free, (c - 1) & 1, ab, false, kBackoffNs)) break;
        load(sm + kScOffW, hb + kHeadOffW, 2 * kWBytes, &w_full);  // W and gamma Q side by side
        ++n_w;
        if (c >= 1 && !mbar_wait(&k_free, (c - 1) & 1, ab, false, kBackoffNs)) break;
        load(sm + kScOffK, kb, kKBytes, &k_full);
        ++n_k;
        if (c >= 1 && !mbar_wait(&p_free, (c - 1) & 1, ab, false, kBackoffNs)) break;
        load(sm + kScOffP, hb + kHeadOffP, 2 * kPImg, &p_full);
        ++n_p;
        if (c + 1 < nc) ok = load_gates(c + 1);
        if (c + 2 < nc) {  // two chunks ahead into L2, behind this chunk's copies
          prefetch_l2(hb + 2LL * p.H_v * kHeadBytes, kHeadBytes);
          prefetch_l2(kb + 2LL * p.H_k * kKBytes, kKBytes);
        }
      }
      // copies still in flight (only possible after an abort) land before the CTA exits
      int drain_flag = 0;
      Abort drain{nullptr, &drain_flag};
      for (int b = 0; b < 2; ++b)
        if (n_g[b] > 0) mbar_wait(&g_full[b], (n_g[b] - 1) & 1, drain);
      if (n_v > 0) mbar_wait(&v_full, (n_v - 1) & 1, drain);
      if (n_bu > 0) mbar_wait(&bu_full, (n_bu - 1) & 1, drain);
      if (n_w > 0) mbar_wait(&w_full, (n_w - 1) & 1, drain);
      if (n_k > 0) mbar_wait(&k_full, (n_k - 1) & 1, drain);
      if (n_p > 0) mbar_wait(&p_full, (n_p - 1) & 1, drain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ output stage (warps 8-11)
    // o = O1 + O2 leaves tensor memory row-wise (thread = d_v row) into shared memory as
    // fp32 [token][d_v], and O is cleared for the next chunk's accumulation; then each thread
    // owns 8 consecutive d_v of a token, 16 threads per token: the sum of o^2 over d_v is a
    // 4-step shuffle inside that group (a fixed order), z is read and out written with
    // 16-byte accesses.
    const int ow = warp & 3;              // TMEM lane quarter
    const int v = 32 * ow + lane;
    const int otid = tid - 256;           // 0..127 within the output group
    const uint32_t tl = tmem_addr(tbase, 32 * ow, 0);
    float* sO = reinterpret_cast<float*>(sm + kScOffO);
    const int v8 = (otid & 15) * 8;       // this thread's 8 channels; its tokens are otid / 16 + 8 m
    float w8[8];  // norm_w is only 2-byte aligned: element loads
#pragma unroll
    for (int e2 = 0; e2 < 8; ++e2) w8[e2] = __bfloat162float(p.norm_w[v8 + e2]);
    mbar_arrive(&o_free);  // the first chunk's state product writes O afresh
    // Every output warp reaches every named barrier; a failed wait is OR-ed into the
    // first barrier so that the four warps leave the loop together.
    for (int c = 0; c < nc; ++c) {
      const long long tok0 = s + static_cast<long long>(c) * kChunk;
      const int L = static_cast<int>(min(static_cast<long long>(kChunk), e - tok0));
      // z of the next chunk into L2 (one 128-byte line per thread), z of this chunk into
      // registers while the products run
      if (c + 1 < nc) {
        const long long r = tok0 + kChunk + (otid >> 1);
        if (r < e) prefetch_l2_line(p.z + r * p.sz + static_cast<long long>(h) * kD + (otid & 1) * 64);
      }
      uint4 zr[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int r = (otid >> 4) + 8 * m;
        zr[m] = r < L ? __ldg(reinterpret_cast<const uint4*>(p.z + (tok0 + r) * p.sz + static_cast<long long>(h) * kD + v8))
                      : make_uint4(0u, 0u, 0u, 0u);
      }
      bool ok = mbar_wait_warp(&y_done, c & 1, ab, false, kBackoffNs);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float o1[32], o2[32];
          tmem_ld32(tl + kColO + 32 * cc, o1);
          tmem_ld32(tl + kColO + 64 + 32 * cc, o2);
          tmem_wait_ld();
          if (cc == 1) {  // O is read: the next chunk's product may overwrite it
            tc_fence_before();
            mbar_arrive(&o_free);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 r = __fadd2_rn(make_float2(o1[i], o1[i + 1]), make_float2(o2[i], o2[i + 1]));
            sO[(32 * cc + i) * kD + v] = r.x;
            sO[(32 * cc + i + 1) * kD + v] = r.y;
          }
        }
      }
      if (bar_sync_or(1, 128, !ok)) break;
      // the eight tokens' sums of squares side by side (independent shuffles), then the outputs
      float inv[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const float4* orow = reinterpret_cast<const float4*>(sO + ((otid >> 4) + 8 * m) * kD + v8);
        const float4 a0 = orow[0], a1 = orow[1];
        float ss = a0.x * a0.x;
        ss = fmaf(a0.y, a0.y, ss); ss = fmaf(a0.z, a0.z, ss); ss = fmaf(a0.w, a0.w, ss);
        ss = fmaf(a1.x, a1.x, ss); ss = fmaf(a1.y, a1.y, ss); ss = fmaf(a1.z, a1.z, ss); ss = fmaf(a1.w, a1.w, ss);
        inv[m] = ss;
      }
#pragma unroll
      for (int sh = 8; sh >= 1; sh >>= 1)
#pragma unroll
        for (int m = 0; m < 8; ++m) inv[m] += __shfl_xor_sync(0xffffffffu, inv[m], sh);
#pragma unroll
      for (int m = 0; m < 8; ++m) inv[m] = rsqrtf(inv[m] * (1.0f / kD) + 1e-6f);
      // two tokens per step, so that their exponential / reciprocal chains overlap
#pragma unroll
      for (int m = 0; m < 8; m += 2) {
        float o8[2][8], y8[2][8], z8[2][8];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float4* orow = reinterpret_cast<const float4*>(sO + ((otid >> 4) + 8 * (m + u)) * kD + v8);
          const float4 a0 = orow[0], a1 = orow[1];
          o8[u][0] = a0.x; o8[u][1] = a0.y; o8[u][2] = a0.z; o8[u][3] = a0.w;
          o8[u][4] = a1.x; o8[u][5] = a1.y; o8[u][6] = a1.z; o8[u][7] = a1.w;
          unpack8(zr[m + u], z8[u]);
        }
#pragma unroll
        for (int e2 = 0; e2 < 8; e2 += 2) {  // ((o inv) w) silu(z), packed in channel pairs
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float2 a = __fmul2_rn(make_float2(o8[u][e2], o8[u][e2 + 1]), make_float2(inv[m + u], inv[m + u]));
            const float2 b = __fmul2_rn(a, make_float2(w8[e2], w8[e2 + 1]));
            const float2 r = __fmul2_rn(b, make_float2(silu_fast(z8[u][e2]), silu_fast(z8[u][e2 + 1])));
            y8[u][e2] = r.x;
            y8[u][e2 + 1] = r.y;
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = (otid >> 4) + 8 * (m + u);
          if (r < L)
            *reinterpret_cast<uint4*>(p.out + ((tok0 + r) * p.H_v + h) * kD + v8) = pack8(y8[u]);
        }
      }
      named_bar_sync(1, 128);  // sO is rewritten by the next chunk
    }
  }

  tc_fence_before();
  named_bar_sync(kScanBar, kScanThreads);
  if (warp == kWarpIssue) tmem_dealloc<512>(tbase);
}

__global__ void __launch_bounds__(kScanThreads, 1) scan_kernel(PrefillParams p) {
  if (p.cu && *p.ws_flag) return;
  extern __shared__ uint8_t scan_smem_raw[];
  scan_body<8>(p, blockIdx.x, align1024(scan_smem_raw));
}

// ------------------------------------------------------------ fused launch
//
// When the scan has few (sequence, value head) CTAs (one long sequence: 48 at 16/48 heads),
// its chain occupies a third of the SMs and the chunk-parallel prep would otherwise run
// first, alone.  One launch then carries both: the last fused_scan_ctas CTAs run the scan
// (448 of their 512 threads; dispatched after the prep CTAs, which measured up to 9% faster
// at 262,144 tokens than scan CTAs first), every other CTA runs two prep items, one per 256-thread half,
// with its own 1024-aligned shared-memory half and 256 of the CTA's 512 tensor-memory
// columns.  Prep items go chunk-major (item = chunk * H_k + key head), so chunks become
// ready in order; the scan's producer waits (bounded) on a chunk's ready flag before its
// first read of that chunk.  No prep CTA waits for anything, and the scan CTAs are at most
// half of the SMs, so the prep always has SMs to run on, in any dispatch order.
constexpr int kFusedThreads = 2 * kPrepThreads;
constexpr int kMaxFusedScanFraction = 2;  // scan CTAs <= SMs / 2
constexpr int kMinFusedItemsPerSm = 8;    // automatic plan: fuse only with >= 8 prep items per prep SM

constexpr int kPrepHalfBytes = (kPrepSmem - 1024 + 1023) / 1024 * 1024;
constexpr int kFusedSmem = 2 * kPrepHalfBytes + 1024 > kScSmem ? 2 * kPrepHalfBytes + 1024 : kScSmem;
static_assert(kFusedThreads >= kScanThreads, "a fused launch's scan CTAs run the scan on their first threads");

__global__ void __launch_bounds__(kFusedThreads, 1) prefill_fused_kernel(PrefillParams p) {
  if (p.cu && *p.ws_flag) return;
  extern __shared__ uint8_t fused_smem_raw[];
  uint8_t* sm = align1024(fused_smem_raw);
  const int first_scan = static_cast<int>(gridDim.x) - p.fused_scan_ctas;
  if (static_cast<int>(blockIdx.x) >= first_scan) {
    // the MMA issue loops rolled: this launch runs the prep's code on the other SMs, and the
    // smaller scan code keeps the two from evicting each other's instructions
    if (threadIdx.x < kScanThreads) scan_body<1>(p, static_cast<int>(blockIdx.x) - first_scan, sm);
    return;
  }
  // prep CTAs: each half is a worker that takes the next item (chunk-major) from a counter in
  // the workspace header until none is left
  __shared__ uint64_t bar[2][4];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s[2];
  __shared__ int go_s;
  __shared__ long long item_s[2];
  const int half = threadIdx.x / kPrepThreads, htid = threadIdx.x & (kPrepThreads - 1);
  const long long n_items = p.n_chunks * p.H_k;
  unsigned long long* counter = reinterpret_cast<unsigned long long*>(p.ws_flag) + 1;
  if (threadIdx.x == 0) go_s = 0;
  if (threadIdx.x < 32) tmem_alloc<512>(&tmem_base_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s + 256u * half;
  uint8_t* smh = sm + half * kPrepHalfBytes;
  if (half == 1 && htid == 0) {
    // start once half 0 is through its first value head (or found nothing to do): the two
    // halves then reach their latency-bound steps at different times
    const long long t0 = clock64();
    while (*reinterpret_cast<volatile int*>(&go_s) == 0 && clock64() - t0 < kWaitLimitCycles) __nanosleep(256);
  }
  for (int k = 0;; ++k) {
    if (htid == 0) item_s[half] = static_cast<long long>(atomicAdd(counter, 1ull));
    named_bar_sync(2 + half, kPrepThreads);
    const long long item = item_s[half];
    if (item >= n_items) {
      if (half == 0 && htid == 0) *reinterpret_cast<volatile int*>(&go_s) = 1;
      break;
    }
    prep_body(p, item / p.H_k, static_cast<int>(item % p.H_k), half, smh, tbase, bar[half], &abort_s[half], k,
              half == 0 && k == 0 ? &go_s : nullptr);
    if (*reinterpret_cast<volatile int*>(&abort_s[half])) break;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) tmem_dealloc<512>(tmem_base_s);
}

// clears the ready flags of every (chunk, value head) before a fused launch
// (and the prep work counter in the workspace header)
__global__ void ready_flags_reset_kernel(PrefillParams p) {
  const long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (x < p.n_chunks * p.H_v) *ready_flag(p, x / p.H_v, static_cast<int>(x % p.H_v)) = 0;
  if (x == 0) reinterpret_cast<unsigned long long*>(p.ws_flag)[1] = 0ull;
}

// SMs this context may run on: the SM resource of the current context (a green context holds
// a partition of the device), scaled down by an MPS active-thread percentage when one is set,
// else the device's count.
int context_sm_count() {
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetResource = CUresult (*)(CUcontext, CUdevResource*, CUdevResourceType);
  static GetCurrent get_current = nullptr;
  static GetResource get_resource = nullptr;
  static const bool have = [] {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetDevResource", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<GetCurrent>(f1);
    get_resource = reinterpret_cast<GetResource>(f2);
    return true;
  }();
  if (have) {
    CUcontext ctx = nullptr;
    CUdevResource res;
    std::memset(&res, 0, sizeof(res));
    if (get_current(&ctx) == CUDA_SUCCESS && ctx && get_resource(ctx, &res, CU_DEV_RESOURCE_TYPE_SM) == CUDA_SUCCESS &&
        res.type == CU_DEV_RESOURCE_TYPE_SM && res.sm.smCount > 0)
      n_sm = std::min(n_sm, static_cast<int>(res.sm.smCount));
  }
  if (const char* pct = std::getenv("CUDA_MPS_ACTIVE_THREAD_PERCENTAGE")) {
    const double f = std::atof(pct);
    if (f > 0.0 && f < 100.0) n_sm = std::max(1, static_cast<int>(n_sm * f / 100.0));
  }
  return n_sm;
}

// the number of scan CTAs of a fused launch, or 0 when the two phases go as two launches:
// gdn_prefill_fused_plan on the context's SMs, if the device also has the shared memory for it
int fused_scan_ctas(const PrefillParams& p) {
  const int schedule = p.allow_fused == 1 ? 0 : p.allow_fused == 2 ? 2 : 1;
  const int n_sm = context_sm_count();
  const int n_scan = gdn_prefill_fused_plan(p.H_k, p.H_v, p.N, p.n_chunks, schedule, n_sm);
  if (n_scan == 0) return 0;
  int dev = 0, smem_optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  cudaFuncAttributes attr;
  if (cudaFuncGetAttributes(&attr, prefill_fused_kernel) != cudaSuccess) return 0;
  if (static_cast<long long>(attr.sharedSizeBytes) + kFusedSmem > smem_optin) return 0;
  return n_scan;
}

cudaError_t launch_scan(const PrefillParams& p, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScSmem);
  if (err != cudaSuccess) return err;
  scan_kernel<<<static_cast<unsigned>(p.N) * p.H_v, kScanThreads, kScSmem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p_in, cudaStream_t stream, void* const* events) {
  cudaError_t err;
  PrefillParams p = p_in;
  p.fused_scan_ctas = fused_scan_ctas(p);
  if (p.cu) {
    setup_kernel<<<1, 1024, 0, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (p.conv_out) {
    const long long C_conv = static_cast<long long>(2 * p.H_k + p.H_v) * kD;
    conv_out_kernel<<<dim3(static_cast<unsigned>((C_conv + 255) / 256), p.N), 256, 0, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (p.fused_scan_ctas > 0) {
    const long long n_flags = p.n_chunks * p.H_v;
    ready_flags_reset_kernel<<<static_cast<unsigned>((n_flags + 255) / 256), 256, 0, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    const int smem = kFusedSmem;
    err = cudaFuncSetAttribute(prefill_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    const long long n_items = p.n_chunks * p.H_k;
    const int n_sm = context_sm_count();
    const long long n_prep = std::min<long long>(n_sm - p.fused_scan_ctas, n_items);
    const unsigned grid = static_cast<unsigned>(p.fused_scan_ctas + n_prep);
    if (events) {  // one launch: the prep / scan split is not observable; [1] sits next to [0]
      cudaEventRecord(static_cast<cudaEvent_t>(events[0]), stream);
      cudaEventRecord(static_cast<cudaEvent_t>(events[1]), stream);
    }
    prefill_fused_kernel<<<grid, kFusedThreads, smem, stream>>>(p);
    err = cudaGetLastError();
    if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[2]), stream);
    return err;
  }
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[0]), stream);
  if (p.n_chunks > 0) {
    const int smem = kPrepSmem;
    err = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    prep_kernel<<<dim3(static_cast<unsigned>(p.n_chunks), p.H_k), kPrepThreads, smem, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
  }
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), stream);
  err = launch_scan(p, stream);
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[2]), stream);
  return err;
}

}  // namespace gdn

extern "C" int gdn_prefill_fused_plan(int H_k, int H_v, int N, long long n_chunks, int schedule, int n_sm) {
  if (H_k <= 0 || H_v <= 0 || N <= 0 || n_chunks <= 0 || n_sm <= 0 || schedule == 1) return 0;
  const long long n_scan = static_cast<long long>(N) * H_v;
  if (n_scan * gdn::kMaxFusedScanFraction > n_sm) return 0;  // the scan CTAs take at most half the SMs
  if (schedule == 0 && n_chunks * H_k < static_cast<long long>(gdn::kMinFusedItemsPerSm) * (n_sm - n_scan)) return 0;
  return static_cast<int>(n_scan);
}
