// The global-attention layer of the hybrid decoder, between its two projections.
//
// Agnes-3.0-Flash model card, "Architecture" table: row "Global attention" (24 query
// heads / 4 KV heads, 6 : 1 GQA, head dim 256, RMS-norm on q and k, sigmoid-gated
// output) and row "Positions" (3-axis rotary, base 1e7, on the first 25 % of each head
// dim = 64 dims); "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model",
// section "Attention Layer Details".  For text tokens the three rotary axes all carry
// the token's position, so every one of the 32 frequencies turns by position * theta_i,
// theta_i = 1e7^(-i/32), applied to the pairs (i, i + 32) of the first 64 dims.
//
// Kernels:
//   attn_qk_kernel     q_hat = rope(rms(q) w_q), k_hat = rope(rms(k) w_k) per head, both
//                      stored bf16 (k_hat into the caller's K cache), v copied to the V cache;
//   flash_attn_kernel  causal softmax attention, GQA, on the tensor cores, with the output
//                      gate o * sigmoid(g) in its epilogue (prefill);
//   attn_decode_kernel, attn_decode_combine_kernel, attn_cache_advance_kernel
//                      one new token per sequence against its KV cache: split-K partials,
//                      their exact merge with the gate, and the cache length update.
#include <cmath>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_kernels.cuh"

namespace gdn {

namespace {

constexpr int kAD = 256;          // head dim
constexpr int kAHq = 24, kAHkv = 4, kAGrp = kAHq / kAHkv;
constexpr int kARope = 64;        // rotary dims per head
constexpr double kARopeBase = 1e7;

// ------------------------------------------------------------ q / k norm and rotary
//
// A warp per 4 (token, head) items of one token: lane l holds dims 8l .. 8l+7 (16-byte loads); the rotary
// pairs (i, i + 32) of dims 0 .. 63 sit in lanes l and l ^ 4 (l < 8).  The angles
// pos * theta_i are formed in fp64 (positions reach 262,144) from frequencies the host
// computes once per launch, reduced to [-pi, pi] by subtracting the nearest multiple of
// 2 pi (one fp64 rounding and fma: error ~1e-10 rad at the largest positions), then sincosf.
constexpr int kQkThreads = 256;
constexpr int kQkItems = 4;  // (token, head) items per warp, all of one token
static_assert((kAHq + 2 * kAHkv) % kQkItems == 0, "a warp's items must belong to one token");
constexpr int kDevErrCacheFull = 16;  // a sequence's KV cache has no row for its new token
constexpr int kDevErrCacheLen = 32;   // a decode cache_len outside [0, cap]: nothing written for that sequence

__device__ __forceinline__ void unpack8f(uint4 u, float* f) {
  f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
  f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ uint4 pack8f(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

struct AttnQkParams {
  const bf16* proj;  // [T_tot][ld_p]: q | g | k | v
  long long ld_p;
  const bf16* q_norm_w;  // [256]
  const bf16* k_norm_w;
  int T;                 // tokens per sequence in this call: token t is number t % T of sequence t / T
  long long T_tot;
  const int* pos_base;   // null (positions 0 .. T-1) or [N]: position of each sequence's first token here
  int cap;               // cache rows per sequence: token at position pos goes to row n * cap + pos
  bf16* q_hat;           // [T_tot][24][256]
  bf16* k_cache;         // [N][cap][4][256]
  bf16* v_cache;         // [N][cap][4][256]
  int* err;
  double theta[kARope / 2];  // rotary frequencies 1e7^(-i/32)
};

__global__ void __launch_bounds__(kQkThreads) attn_qk_kernel(AttnQkParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kHeads = kAHq + kAHkv + kAHkv;  // q heads, k heads, v heads
  const long long n_items = p.T_tot * kHeads;
  // a warp takes kQkItems consecutive (token, head) items of one token and issues their loads together
  const long long item0 = (static_cast<long long>(blockIdx.x) * (kQkThreads / 32) + warp) * kQkItems;
  if (item0 >= n_items) return;  // warp-uniform
  uint4 raw[kQkItems];
#pragma unroll
  for (int u = 0; u < kQkItems; ++u) {
    const long long item = item0 + u;
    raw[u] = make_uint4(0u, 0u, 0u, 0u);
    if (item < n_items) {
      const long long t = item / kHeads;
      const int hh = static_cast<int>(item % kHeads);
      const bf16* row = p.proj + t * p.ld_p;
      const bf16* src = hh < kAHq ? row + hh * kAD : row + 2 * kAHq * kAD + (hh - kAHq) * kAD;  // k and v follow g
      raw[u] = reinterpret_cast<const uint4*>(src)[lane];
    }
  }
  float wq[8], wk[8];
  unpack8f(reinterpret_cast<const uint4*>(p.q_norm_w)[lane], wq);
  unpack8f(reinterpret_cast<const uint4*>(p.k_norm_w)[lane], wk);
  // the rotation of this token, shared by its heads: lane i turns frequency i (its angle formed in
  // fp64 and reduced to [-pi, pi]), then lanes 0..7 gather the 8 frequencies 8 (l % 4) + e they apply
  const long long t_w = item0 / kHeads;
  const long long pos_w = (p.pos_base ? p.pos_base[t_w / p.T] : 0) + t_w % p.T;
  float cs8[8], sn8[8];
  {
    constexpr double kTwoPi = 6.283185307179586476925286766559, kInvTwoPi = 0.15915494309189533576888376337251;
    const double ang = static_cast<double>(pos_w) * p.theta[lane];
    const double r = fma(-rint(ang * kInvTwoPi), kTwoPi, ang);
    float sn, cs;
    sincosf(static_cast<float>(r), &sn, &cs);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cs8[e] = __shfl_sync(0xffffffffu, cs, 8 * (lane & 3) + e);
      sn8[e] = __shfl_sync(0xffffffffu, sn, 8 * (lane & 3) + e);
    }
  }
#pragma unroll
  for (int u = 0; u < kQkItems; ++u) {
    const long long item = item0 + u;
    if (item >= n_items) continue;  // warp-uniform
    const long long t = item / kHeads;
    const int hh = static_cast<int>(item % kHeads);
    const long long n = t / p.T;
    const long long pos = (p.pos_base ? p.pos_base[n] : 0) + t % p.T;
    if (pos < 0 || pos >= p.cap) {  // no room in the cache, or a bad length: nothing is written for it
      if (lane == 0 && hh == 0 && p.err) atomicOr(p.err, pos == p.cap ? kDevErrCacheFull : kDevErrCacheLen);
      continue;
    }
    const long long crow = n * p.cap + pos;  // cache row of this token
    if (hh >= kAHq + kAHkv) {  // v: a copy into the cache
      reinterpret_cast<uint4*>(p.v_cache + (crow * kAHkv + (hh - kAHq - kAHkv)) * kAD)[lane] = raw[u];
      continue;
    }
    const bool is_q = hh < kAHq;
    const int h = is_q ? hh : hh - kAHq;
    float x[8];
    unpack8f(raw[u], x);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss * (1.0f / kAD) + 1e-6f);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = x[e] * inv * (is_q ? wq[e] : wk[e]);
    // rotary on dims 0 .. 63 (lanes 0 .. 7): lane l < 4 holds x1 = dims 8l.., lane l + 4 holds x2
    float partner[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) partner[e] = __shfl_xor_sync(0xffffffffu, x[e], 4);
    if (lane < 8) {
#pragma unroll
      for (int e = 0; e < 8; ++e)  // x1' = x1 c - x2 s (lanes 0..3), x2' = x2 c + x1 s (lanes 4..7)
        x[e] = lane < 4 ? fmaf(x[e], cs8[e], -partner[e] * sn8[e]) : fmaf(x[e], cs8[e], partner[e] * sn8[e]);
    }
    bf16* dst = is_q ? p.q_hat + (t * kAHq + h) * kAD : p.k_cache + (crow * kAHkv + h) * kAD;
    reinterpret_cast<uint4*>(dst)[lane] = pack8f(x);
  }
}

// ------------------------------------------------------------ causal flash attention
//
// One CTA per (query tile of 128 tokens, query head); tiles of one sequence go longest
// first.  Warps 0-7: softmax and epilogue (thread = query row, TMEM lane quarter = warp % 4;
// warps w and w + 4 split the row's 128 score columns and O's 256 columns in halves and
// trade their partial row maxima through shared memory); warp 8 lanes 0 / 1: TMA (Q once
// and the K tiles / the V tiles of 128 keys, one buffer each); warp 9 lane 0: tcgen05.mma.
// Per key tile j:
//   S_j  = Q K_j^T            M 128, N 128, K 256  (16 MMAs; A, B K-major from shared memory)
//   P_j  = exp2(S_j log2(e)/16 - m)                (softmax warps; bf16 pairs written over the
//                                                   first 64 columns of S_j's own TMEM buffer)
//   O   += P_j V_j            M 128, N 256, K 128  (8 MMAs; A = P from TMEM, B = V MN-major)
// TMEM: O in columns 0..255, S in two buffers of 128 columns, so S_{j+1} runs while the
// softmax works on S_j; S_{j+2} reuses S_j's buffer once O += P_j V_j has read P_j.  The next
// K tile loads as soon as S_j has read K_j, the next V tile once P_j V_j has read V_j.  The
// running max is lazy: O and l are rescaled only when a row's max grows by more than 8
// (log2 units), decided per warp (the wait and the TMEM accesses are warp-collective), after
// the products still writing O; the final 1/l makes the result exact either way.  Masked
// scores (key past the query) are -inf.  Epilogue: o / l * sigmoid(g) in bf16 into
// [T_tot][24 * 256].  Every wait is bounded.
constexpr int kFaBM = 128, kFaBN = 128;
constexpr int kFaThreads = 320;
constexpr int kFaWarpTma = 8, kFaWarpMma = 9;
constexpr int kFaQBytes = kFaBM * kAD * 2;          // 64 KiB: 4 boxes of 128 rows x 64 dims
constexpr int kFaKBytes = kFaBN * kAD * 2;          // 64 KiB: 4 boxes of 128 keys x 64 dims
constexpr int kFaSmem = kFaQBytes + 2 * kFaKBytes + 1024;  // Q | K | V
// tensor memory columns
constexpr uint32_t kFaColO = 0;      // 256 fp32 columns
constexpr uint32_t kFaColS = 256;    // 2 x 128 (P of the tile in the first 64 of its buffer)
constexpr float kFaRescale = 8.0f;   // lazy rescale threshold (log2 units)

struct FaParams {
  int T;              // tokens per sequence
  int B;              // sequences
  // K, V: 3-D tensor maps (columns, T rows, B sequences at a stride of the cache capacity), so
  // rows past a sequence's T tokens read as zeros, whatever the cache holds there
  int tiles;          // query tiles per sequence
  const bf16* g;      // gate: head h of token t at g + t * ld_g + h * 256
  long long ld_g;
  bf16* out;          // [T_tot][24*256]
  int* err;
  float scale_log2e;  // log2(e) / sqrt(256)
};

__device__ __forceinline__ uint8_t* fa_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void fa_tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled TMA load of the box at (x = column, y = row, z = sequence)
__device__ __forceinline__ void fa_tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                               uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kFaThreads, 1)
    flash_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, FaParams p) {
  extern __shared__ uint8_t fa_smem_raw[];
  uint8_t* sm = fa_align1024(fa_smem_raw);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + kFaQBytes;
  uint8_t* sV = sK + kFaKBytes;
  __shared__ uint64_t q_full, k_full, k_free, v_full, v_free, s_full[2], p_full[2], pv_done[2], drain_b;
  __shared__ float red_s[2][kFaBM];  // partial row maxima (and at the end partial sums), per column half
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: head h, sequence n, query tile mt (longest tiles first)
  const int h = blockIdx.y;
  const int n = blockIdx.x % p.B;
  const int mt = p.tiles - 1 - static_cast<int>(blockIdx.x / p.B);
  const int m0 = mt * kFaBM;                                  // first query position in the sequence
  const int n_kv = (min(m0 + kFaBM, p.T) + kFaBN - 1) / kFaBN;  // key tiles (causal)
  const int kvh = h / kAGrp;
  const int row0 = n * p.T;                                   // first token of the sequence

  const Abort ab{p.err, &abort_s};
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&q_full, 1);
    mbar_init(&k_full, 1);
    mbar_init(&k_free, 1);
    mbar_init(&v_full, 1);
    mbar_init(&v_free, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(&drain_b, 1);
    fence_mbar_init();
  }
  if (warp == kFaWarpMma) tmem_alloc<512>(&tmem_base_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base_s;

  if (warp == kFaWarpTma) {
    // ------------------------------------------------ TMA producers: lane 0 Q and the K tiles,
    // lane 1 the V tiles, each waiting only for its own buffer
    int drain_flag = 0;
    const Abort drain{nullptr, &drain_flag};
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, kFaQBytes);
      for (int kb = 0; kb < 4; ++kb)
        fa_tma_load_2d(sQ + kb * (kFaBM * 128), &tm_q, h * kAD + kb * 64, row0 + m0, &q_full);
      int n_k = 0;
      for (int j = 0; j < n_kv; ++j) {  // K_j once S_{j-1} has read K_{j-1}
        if (j >= 1 && !mbar_wait(&k_free, (j - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&k_full, kFaKBytes);
        for (int kb = 0; kb < 4; ++kb)
          fa_tma_load_3d(sK + kb * (kFaBN * 128), &tm_k, kvh * kAD + kb * 64, j * kFaBN, n, &k_full);
        ++n_k;
      }
      // copies still in flight (only after an abort) land before the CTA exits
      mbar_wait(&q_full, 0, drain);
      if (n_k > 0) mbar_wait(&k_full, (n_k - 1) & 1, drain);
    } else if (lane == 1) {
      int n_v = 0;
      for (int j = 0; j < n_kv; ++j) {  // V_j once P_{j-1} V_{j-1} has read V_{j-1}
        if (j >= 1 && !mbar_wait(&v_free, (j - 1) & 1, ab)) break;
        mbar_arrive_expect_tx(&v_full, kFaKBytes);
        for (int kb = 0; kb < 4; ++kb)
          fa_tma_load_3d(sV + kb * (kFaBN * 128), &tm_v, kvh * kAD + kb * 64, j * kFaBN, n, &v_full);
        ++n_v;
      }
      if (n_v > 0) mbar_wait(&v_full, (n_v - 1) & 1, drain);
    }
  } else if (warp == kFaWarpMma) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc_s = idesc_bf16(kFaBM, kFaBN, false, false);  // Q K^T
      const uint32_t idesc_o = idesc_bf16(kFaBM, kAD, false, true);     // P V, V MN-major (N = d)
      const uint32_t q_s = smem_u32(sQ), k_s = smem_u32(sK), v_s = smem_u32(sV);
      bool ok = mbar_wait(&q_full, 0, ab);
      auto issue_pv = [&](int i) -> bool {  // O += P_i V_i
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, ab)) return false;
        if (!mbar_wait(&v_full, i & 1, ab)) return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kFaBN / 16; ++ks)
          umma_bf16_ts(tbase + kFaColO, tbase + kFaColS + 128u * (i & 1) + 8u * ks,
                       smem_desc(v_s + ks * 2048u, kFaBN * 128, 1024, Swz::k128), idesc_o, i > 0 || ks > 0);
        umma_commit(&pv_done[i & 1]);
        umma_commit(&v_free);
        return true;
      };
      for (int j = 0; j < n_kv && ok; ++j) {
        const int s = j & 1;
        if (!mbar_wait(&k_full, j & 1, ab)) break;
        // S buffer s held P_{j-2}: its products must have read it
        if (j >= 2 && !mbar_wait(&pv_done[s], ((j - 2) >> 1) & 1, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kAD / 16; ++ks) {
          const uint32_t off_q = (ks >> 2) * (kFaBM * 128u) + (ks & 3) * 32u;
          const uint32_t off_k = (ks >> 2) * (kFaBN * 128u) + (ks & 3) * 32u;
          umma_bf16(tbase + kFaColS + 128u * s, smem_desc(q_s + off_q, 16, 1024, Swz::k128),
                    smem_desc(k_s + off_k, 16, 1024, Swz::k128), idesc_s, ks > 0);
        }
        umma_commit(&s_full[s]);
        umma_commit(&k_free);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n_kv > 0) issue_pv(n_kv - 1);
      umma_commit(&drain_b);
      int drain_flag = 0;
      const Abort drain{nullptr, &drain_flag};
      mbar_wait(&drain_b, 0, drain);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue: thread = query row,
    // column half hc of the scores (keys 64 hc ..) and of O (d 128 hc ..)
    const int q4 = warp & 3, hc = warp >> 2;
    const int r = 32 * q4 + lane;
    const int qpos = m0 + r;
    const uint32_t trow = tmem_addr(tbase, 32 * q4, 0);
    constexpr int kHalf = kFaBN / 2;  // 64 score columns per thread
    float m = -INFINITY, l = 0.f;     // l: this half's partial sum
    // no early exit: the two warps of a row pair meet at named barriers every tile, so after a
    // failed wait a warp keeps its place in the loop and only skips its tensor-memory work
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      ok = ok && mbar_wait_warp(&s_full[s], (j >> 1) & 1, ab);
      tc_fence_after();
      float sv[kHalf];
      if (ok) {
        tmem_ld32(trow + kFaColS + 128u * s + kHalf * hc, sv);
        tmem_ld32(trow + kFaColS + 128u * s + kHalf * hc + 32u, sv + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < kHalf; ++c) sv[c] = 0.f;
      }
      const int k0 = j * kFaBN + kHalf * hc;
      float mraw = -INFINITY;  // max of the raw scores (the scale is positive)
      if (k0 + kHalf - 1 <= m0) {  // no key of this half lies past any query of the tile
#pragma unroll
        for (int c = 0; c < kHalf; ++c) mraw = fmaxf(mraw, sv[c]);
      } else {
#pragma unroll
        for (int c = 0; c < kHalf; ++c) {
          sv[c] = (k0 + c <= qpos) ? sv[c] : -INFINITY;
          mraw = fmaxf(mraw, sv[c]);
        }
      }
      // the row's max from both halves
      red_s[hc][r] = mraw;
      named_bar_sync(1 + q4, 64);
      const float mloc = fmaxf(mraw, red_s[hc ^ 1][r]) * p.scale_log2e;
      named_bar_sync(1 + q4, 64);  // both have read before the next tile's write
      // the rescale is decided per warp (the wait and the TMEM accesses are warp-collective);
      // both warps of a row pair see the same maxima, so they decide alike
      const bool grow = mloc > m + kFaRescale;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = grow ? mloc : m;
        if (j >= 1) {
          // rescale the warp's half of its rows of O once the products of tile j - 1 have written them
          ok = ok && mbar_wait_warp(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, ab);
        }
        if (j >= 1 && ok) {
          tc_fence_after();
          const float f = exp2f(m - m_new);  // 1 for lanes keeping their max
#pragma unroll 1
          for (int c = 0; c < kAD / 64; ++c) {
            float o[32];
            tmem_ld32(trow + kFaColO + 128u * hc + 32u * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= f;
            tmem_st32(trow + kFaColO + 128u * hc + 32u * c, o);
          }
          l *= f;
        }
        m = m_new;
      }
      uint32_t pk[kHalf / 2];
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < kHalf / 2; ++c) {
        const float p0 = exp2f(fmaf(sv[2 * c], p.scale_log2e, -m));
        const float p1 = exp2f(fmaf(sv[2 * c + 1], p.scale_log2e, -m));
        lsum += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l += lsum;
      if (ok) {
        tmem_st16(trow + kFaColS + 128u * s + 32u * hc, pk);
        tmem_st16(trow + kFaColS + 128u * s + 32u * hc + 16u, pk + 16);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[s]);
      }
    }
    // epilogue: the last tile's products complete every write to O; l from both halves
    red_s[hc][r] = l;
    named_bar_sync(1 + q4, 64);
    const float l_row = l + red_s[hc ^ 1][r];
    if (ok && n_kv > 0 && mbar_wait_warp(&pv_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, ab)) {
      tc_fence_after();
      const bool valid = qpos < p.T;
      const long long tok = static_cast<long long>(row0) + qpos;
      const float inv_l = 1.0f / l_row;
      const bf16* grow_p = p.g + tok * p.ld_g + h * kAD + 128 * hc;
      bf16* orow = p.out + tok * (kAHq * kAD) + h * kAD + 128 * hc;
#pragma unroll 1
      for (int c = 0; c < kAD / 64; ++c) {
        float o[32];
        tmem_ld32(trow + kFaColO + 128u * hc + 32u * c, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float gf[8], y[8];
            unpack8f(reinterpret_cast<const uint4*>(grow_p + 32 * c)[u], gf);
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = o[8 * u + e] * inv_l / (1.0f + __expf(-gf[e]));
            reinterpret_cast<uint4*>(orow + 32 * c)[u] = pack8f(y);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kFaWarpMma) tmem_dealloc<512>(tbase);
}

// ------------------------------------------------------------ decode over the KV cache
//
// One new token per sequence, already appended to the cache by attn_qk_kernel (at row
// cache_len[n]); its 24 queries attend to rows 0 .. cache_len[n].  Split-K: CTA (split, KV
// head, sequence) takes up to kDecSplit cache rows and the KV head's 6 query heads, in fp32
// accumulation.  Both contractions run on the tensor cores as m16n8k16 bf16 MMAs (warp-level:
// the 6 heads are far below the 64-row minimum of a tcgen05 tile), which leaves the CUDA cores
// only the softmax; the kernel is HBM-bound by design (the cache is read once per KV head per
// step).  attn_decode_combine_kernel merges the splits per (sequence, query head), applies 1/l
// and sigmoid(g) and writes bf16; a last small kernel advances cache_len.
constexpr int kDecSplit = 512;   // cache rows per CTA (a multiple of 128)
constexpr int kDecThreads = 256;
constexpr int kDecPart = kAD + 2;  // o[256], m, l

struct AttnDecParams {
  const bf16* q_hat;      // [N][24][256]
  const bf16* k_cache;    // [N][cap][4][256]
  const bf16* v_cache;
  int cap;
  const int* cache_len;   // [N] rows before this step; the new token sits at row cache_len[n]
  int n_splits;
  float* part;            // [N][4][n_splits][6][kDecPart]
};

// d (16 x 8 fp32) += A (16 x 16 bf16, row-major fragment a) B (16 x 8 bf16, column fragment b):
// lane (g = lane / 4, c = lane % 4) holds A rows g, g + 8 at columns 2c, 2c + 1 (a0, a1) and
// 2c + 8, 2c + 9 (a2, a3), B column g at rows 2c, 2c + 1 (b0) and 2c + 8, 2c + 9 (b1), and
// D rows g (d0, d1), g + 8 (d2, d3) at columns 2c, 2c + 1.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kDecThreads, 2) attn_decode_kernel(AttnDecParams p) {
  const int sp = blockIdx.x, kvh = blockIdx.y, n = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  __shared__ float sc[kAGrp][kDecSplit];
  __shared__ float os[kAGrp][kAD];
  __shared__ float mh[kAGrp], lh[kAGrp];
  float* part = p.part + ((static_cast<long long>(n) * kAHkv + kvh) * p.n_splits + sp) * kAGrp * kDecPart;
  const int len = p.cache_len[n] + 1;
  const int t0 = sp * kDecSplit, t1 = min(t0 + kDecSplit, len);
  if (len <= 0 || len > p.cap || t0 >= t1) {  // nothing here (no room, or a bad length): an empty partial
    if (threadIdx.x < kAGrp) {
      part[threadIdx.x * kDecPart + kAD] = -INFINITY;
      part[threadIdx.x * kDecPart + kAD + 1] = 0.f;
    }
    return;
  }
  for (int x = threadIdx.x; x < kAGrp * kAD; x += kDecThreads) os[x / kAD][x % kAD] = 0.f;
  const long long row_el = static_cast<long long>(kAHkv) * kAD;  // elements between cache rows
  const bf16* kbase = p.k_cache + (static_cast<long long>(n) * p.cap * kAHkv + kvh) * kAD;
  const bf16* vbase = p.v_cache + (static_cast<long long>(n) * p.cap * kAHkv + kvh) * kAD;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);

  // pass 1: S[token][head] = K q^T, M = 16 tokens, N = 8 heads (6 used), K = 256 dims in 16
  // MMAs.  The dot product does not depend on the order of the dims, so MMA 2m + h gives lane
  // (g, c)'s four k slots {2c, 2c+1, 2c+8, 2c+9} the dims 8 (4m + c) + 4h + {0, 1, 2, 3}: each
  // lane's operands are then whole 16-byte pieces of a K row (dims 8 (4m + c) .. + 7) and of its
  // query head g, loaded straight into fragment order.  Warp w scores the 16-token blocks
  // t0 + 16 (w + 8 blk); the two halves of the dims accumulate separately (shorter MMA chains).
  {
    uint4 qf[8];
    const uint4* qrow = reinterpret_cast<const uint4*>(
        p.q_hat + (static_cast<long long>(n) * kAHq + kvh * kAGrp + min(g, kAGrp - 1)) * kAD);
#pragma unroll
    for (int m = 0; m < 8; ++m) qf[m] = g < kAGrp ? qrow[4 * m + c] : zero4;
#pragma unroll 1
    for (int blk = 0; blk < kDecSplit / 128; ++blk) {
      const int tb = t0 + 16 * (warp + 8 * blk);
      if (tb >= t1) break;  // warp-uniform
      const int r0 = tb + g, r1 = tb + g + 8;
      const uint4* k0 = reinterpret_cast<const uint4*>(kbase + r0 * row_el);
      const uint4* k1 = reinterpret_cast<const uint4*>(kbase + r1 * row_el);
      uint4 a0[8], a1[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        a0[m] = r0 < t1 ? k0[4 * m + c] : zero4;
        a1[m] = r1 < t1 ? k1[4 * m + c] : zero4;
      }
      float s4[4] = {0.f, 0.f, 0.f, 0.f}, t4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        mma_16816(s4, a0[m].x, a1[m].x, a0[m].y, a1[m].y, qf[m].x, qf[m].y);
        mma_16816(t4, a0[m].z, a1[m].z, a0[m].w, a1[m].w, qf[m].z, qf[m].w);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) s4[e] += t4[e];
      if (c < kAGrp / 2) {  // heads 2c, 2c + 1; scores scaled by 1/sqrt(256)
        if (r0 < t1) {
          sc[2 * c][r0 - t0] = s4[0] * 0.0625f;
          sc[2 * c + 1][r0 - t0] = s4[1] * 0.0625f;
        }
        if (r1 < t1) {
          sc[2 * c][r1 - t0] = s4[2] * 0.0625f;
          sc[2 * c + 1][r1 - t0] = s4[3] * 0.0625f;
        }
      }
    }
  }

  // pass 2 operands.  O^T[dim][head] += V^T[dim][token] P^T[token][head]: M = 16 dims, N = 8
  // heads, K = 16 tokens.  Warp pair wp = warp / 2 takes the 32-token groups t0 + 32 (wp + 4 it), warp
  // parity dh the dims 128 dh .. + 127.  Lane (g, c) holds tokens 2c, 2c+1, 2c+8, 2c+9 of a 16-token
  // block (slots u = 0..3) and, for each, the two 16-byte pieces at dims 128 dh + 8g and
  // 128 dh + 64 + 8g; tile i (0..7) takes 32-bit word i of those 8: dims D_i, D_i + 1 as its
  // rows g, g + 8, with the token pairs formed by byte permutes.  The pair's first 32-token group's loads
  // are issued before the softmax.
  const int dh = warp & 1, wp = warp >> 1;
  const int tv0 = t0 + 32 * wp;
  uint4 vr[2][4][2];
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = tv0 + 16 * b + 2 * c + (u & 1) + 8 * (u >> 1);
      const uint4* row = reinterpret_cast<const uint4*>(vbase + t * row_el + 128 * dh + 8 * g);
      vr[b][u][0] = t < t1 ? row[0] : zero4;
      vr[b][u][1] = t < t1 ? row[8] : zero4;
    }
  __syncthreads();
  // per-head max, exponentials and sum (warp j < 6 takes head j); slots past the split's last
  // token become 0 so that pass 2 reads no stale values
  if (warp < kAGrp) {
    const int cnt = t1 - t0;
    float m = -INFINITY;
    for (int i = lane; i < cnt; i += 32) m = fmaxf(m, sc[warp][i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int i = lane; i < kDecSplit; i += 32) {
      const float e = i < cnt ? expf(sc[warp][i] - m) : 0.f;
      sc[warp][i] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      mh[warp] = m;
      lh[warp] = l;
    }
  }
  __syncthreads();
  // pass 2: the weights p as a bf16 pair p_hi + p_lo (two MMAs), about 16 significant bits
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const float* prow = &sc[min(g, kAGrp - 1)][0];
#pragma unroll 1
  for (int it = 0; it < kDecSplit / 128; ++it) {
    const int tb = tv0 + 128 * it;
    if (tb >= t1) break;  // warp-uniform
    if (it > 0) {
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = tb + 16 * b + 2 * c + (u & 1) + 8 * (u >> 1);
          const uint4* row = reinterpret_cast<const uint4*>(vbase + t * row_el + 128 * dh + 8 * g);
          vr[b][u][0] = t < t1 ? row[0] : zero4;
          vr[b][u][1] = t < t1 ? row[8] : zero4;
        }
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int tr = tb + 16 * b - t0 + 2 * c;  // this lane's first token, relative to t0
      float2 p01 = *reinterpret_cast<const float2*>(prow + tr);
      float2 p89 = *reinterpret_cast<const float2*>(prow + tr + 8);
      if (g >= kAGrp) p01 = p89 = make_float2(0.f, 0.f);
      const uint32_t b0h = pack_bf16x2(p01.x, p01.y), b1h = pack_bf16x2(p89.x, p89.y);
      const uint32_t b0l = pack_bf16x2(p01.x - bf16_lo(b0h), p01.y - bf16_hi(b0h));
      const uint32_t b1l = pack_bf16x2(p89.x - bf16_lo(b1h), p89.y - bf16_hi(b1h));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w0 = (&vr[b][0][i >> 2].x)[i & 3], w1 = (&vr[b][1][i >> 2].x)[i & 3];
        const uint32_t w8 = (&vr[b][2][i >> 2].x)[i & 3], w9 = (&vr[b][3][i >> 2].x)[i & 3];
        const uint32_t x0 = __byte_perm(w0, w1, 0x5410), x1 = __byte_perm(w0, w1, 0x7632);
        const uint32_t x2 = __byte_perm(w8, w9, 0x5410), x3 = __byte_perm(w8, w9, 0x7632);
        mma_16816(acc[i], x0, x1, x2, x3, b0h, b1h);
        mma_16816(acc[i], x0, x1, x2, x3, b0l, b1l);
      }
    }
  }
  // the four warp pairs' partial sums of each (head, dim)
  if (c < kAGrp / 2) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int d = 128 * dh + 64 * (i >> 2) + 8 * g + 2 * (i & 3);
      atomicAdd(&os[2 * c][d], acc[i][0]);
      atomicAdd(&os[2 * c + 1][d], acc[i][1]);
      atomicAdd(&os[2 * c][d + 1], acc[i][2]);
      atomicAdd(&os[2 * c + 1][d + 1], acc[i][3]);
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < kAGrp * kAD; x += kDecThreads) part[(x / kAD) * kDecPart + x % kAD] = os[x / kAD][x % kAD];
  if (threadIdx.x < kAGrp) {
    part[threadIdx.x * kDecPart + kAD] = mh[threadIdx.x];
    part[threadIdx.x * kDecPart + kAD + 1] = lh[threadIdx.x];
  }
}

// merge the splits of (sequence n, query head h): o = sum_s o_s e^{m_s - M} / sum_s l_s e^{m_s - M}.
// The splits' weights e^{m_s - M} are formed once per CTA in shared memory (kDecMergeMax splits at
// a time), then each thread (one output dim) sums its column with four loads in flight.
constexpr int kDecMergeMax = 512;
__global__ void __launch_bounds__(kAD) attn_decode_combine_kernel(AttnDecParams p, const bf16* g, long long ld_g,
                                                                  bf16* out) {
  const int n = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int kvh = h / kAGrp, j = h % kAGrp;
  __shared__ float w_s[kDecMergeMax];
  __shared__ float red_s[kAD / 32];
  const int len = p.cache_len[n] + 1;
  if (len <= 0 || len > p.cap) {  // reported by the cache write; nothing was attended: a zero output row
    out[(static_cast<long long>(n) * kAHq + h) * kAD + d] = __float2bfloat16(0.f);
    return;
  }
  const int used = (len + kDecSplit - 1) / kDecSplit;
  const float* base = p.part + (static_cast<long long>(n) * kAHkv + kvh) * p.n_splits * kAGrp * kDecPart;
  // M = max over the splits of m_s
  float M = -INFINITY;
  for (int s2 = d; s2 < used; s2 += kAD) M = fmaxf(M, base[(s2 * kAGrp + j) * kDecPart + kAD]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if ((d & 31) == 0) red_s[d >> 5] = M;
  __syncthreads();
  M = red_s[0];
#pragma unroll
  for (int w = 1; w < kAD / 32; ++w) M = fmaxf(M, red_s[w]);
  float O = 0.f, L = 0.f;
  for (int c0 = 0; c0 < used; c0 += kDecMergeMax) {
    const int cn = min(kDecMergeMax, used - c0);
    __syncthreads();  // red_s and w_s are free
    float Lp = 0.f;
    for (int s2 = d; s2 < cn; s2 += kAD) {
      const float* ps = base + ((c0 + s2) * kAGrp + j) * kDecPart;
      const float w = expf(ps[kAD] - M);
      w_s[s2] = w;
      Lp = fmaf(ps[kAD + 1], w, Lp);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Lp += __shfl_xor_sync(0xffffffffu, Lp, o);
    if ((d & 31) == 0) red_s[d >> 5] = Lp;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kAD / 32; ++w) L += red_s[w];
    const float* col = base + (static_cast<long long>(c0) * kAGrp + j) * kDecPart + d;
    int s2 = 0;
    for (; s2 + 4 <= cn; s2 += 4) {
      const float o0 = col[(s2 + 0) * kAGrp * kDecPart], o1 = col[(s2 + 1) * kAGrp * kDecPart];
      const float o2 = col[(s2 + 2) * kAGrp * kDecPart], o3 = col[(s2 + 3) * kAGrp * kDecPart];
      O = fmaf(o0, w_s[s2], O);
      O = fmaf(o1, w_s[s2 + 1], O);
      O = fmaf(o2, w_s[s2 + 2], O);
      O = fmaf(o3, w_s[s2 + 3], O);
    }
    for (; s2 < cn; ++s2) O = fmaf(col[s2 * kAGrp * kDecPart], w_s[s2], O);
  }
  const float gv = __bfloat162float(g[static_cast<long long>(n) * ld_g + h * kAD + d]);
  out[(static_cast<long long>(n) * kAHq + h) * kAD + d] = __float2bfloat16(O / L / (1.0f + expf(-gv)));
}

// the step is complete: each sequence's cache holds one more row (unless it was full)
__global__ void attn_cache_advance_kernel(int* cache_len, int N, int cap) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N && cache_len[n] >= 0 && cache_len[n] < cap) cache_len[n] += 1;
}

PFN_cuTensorMapEncodeTiled_v12000 attn_map_encoder() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

// bf16 [rows][ld] as 64-column x box_rows boxes, 128-byte swizzle, zero fill past the edges
bool attn_encode(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, long long rows,
                 long long cols, long long ld, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 cache [B][cap][cols]: the first T rows of each sequence as 64-column x box_rows x 1 boxes
bool attn_encode_cache(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* map, const void* base, int B, int T,
                       int cap, long long cols, int box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, static_cast<cuuint64_t>(cap) * cols * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_qk(const bf16* proj, long long ld_p, const bf16* q_norm_w, const bf16* k_norm_w, int B,
                           int T, const int* pos_base, int cap, bf16* q_hat, bf16* k_cache, bf16* v_cache, int* err,
                           cudaStream_t stream) {
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot == 0) return cudaSuccess;
  AttnQkParams qp;
  qp.proj = proj;
  qp.ld_p = ld_p;
  qp.q_norm_w = q_norm_w;
  qp.k_norm_w = k_norm_w;
  qp.T = T;
  qp.T_tot = T_tot;
  qp.pos_base = pos_base;
  qp.cap = cap;
  qp.q_hat = q_hat;
  qp.k_cache = k_cache;
  qp.v_cache = v_cache;
  qp.err = err;
  for (int i = 0; i < kARope / 2; ++i) qp.theta[i] = std::pow(kARopeBase, -static_cast<double>(i) / (kARope / 2));
  const long long items = T_tot * (kAHq + 2 * kAHkv);
  const long long per_cta = static_cast<long long>(kQkThreads / 32) * kQkItems;
  attn_qk_kernel<<<static_cast<unsigned>((items + per_cta - 1) / per_cta), kQkThreads, 0, stream>>>(qp);
  return cudaGetLastError();
}

cudaError_t launch_flash_attn(const bf16* q_hat, const bf16* k, const bf16* v, int kv_cap, const bf16* g,
                              long long ld_g, int B, int T, bf16* out, int* err, cudaStream_t stream) {
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot == 0) return cudaSuccess;
  PFN_cuTensorMapEncodeTiled_v12000 enc = attn_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  if (!attn_encode(enc, &tq, q_hat, T_tot, kAHq * kAD, kAHq * kAD, kFaBM) ||
      !attn_encode_cache(enc, &tk, k, B, T, kv_cap, kAHkv * kAD, kFaBN) ||
      !attn_encode_cache(enc, &tv, v, B, T, kv_cap, kAHkv * kAD, kFaBN))
    return cudaErrorInvalidValue;
  FaParams fp;
  fp.T = T;
  fp.B = B;
  fp.tiles = (T + kFaBM - 1) / kFaBM;
  fp.g = g;
  fp.ld_g = ld_g;
  fp.out = out;
  fp.err = err;
  fp.scale_log2e = 1.4426950408889634f / 16.0f;  // log2(e) / sqrt(256)
  cudaError_t e = cudaFuncSetAttribute(flash_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFaSmem);
  if (e != cudaSuccess) return e;
  flash_attn_kernel<<<dim3(static_cast<unsigned>(fp.tiles * B), kAHq), kFaThreads, kFaSmem, stream>>>(tq, tk, tv, fp);
  return cudaGetLastError();
}

int attn_decode_splits(int cap) { return (cap + kDecSplit - 1) / kDecSplit; }

size_t attn_decode_part_bytes(int N, int cap) {
  return static_cast<size_t>(N) * kAHkv * attn_decode_splits(cap) * kAGrp * kDecPart * sizeof(float);
}

cudaError_t launch_attn_decode(const bf16* q_hat, const bf16* k_cache, const bf16* v_cache, int cap, int* cache_len,
                               const bf16* g, long long ld_g, int N, float* part, bf16* out, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  AttnDecParams dp;
  dp.q_hat = q_hat;
  dp.k_cache = k_cache;
  dp.v_cache = v_cache;
  dp.cap = cap;
  dp.cache_len = cache_len;
  dp.n_splits = attn_decode_splits(cap);
  dp.part = part;
  attn_decode_kernel<<<dim3(static_cast<unsigned>(dp.n_splits), kAHkv, static_cast<unsigned>(N)), kDecThreads, 0,
                       stream>>>(dp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<<<dim3(static_cast<unsigned>(N), kAHq), kAD, 0, stream>>>(dp, g, ld_g, out);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  attn_cache_advance_kernel<<<(N + 127) / 128, 128, 0, stream>>>(cache_len, N, cap);
  return cudaGetLastError();
}

}  // namespace gdn
