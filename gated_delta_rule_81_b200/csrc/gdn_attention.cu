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
// Two kernels:
//   attn_qk_kernel     q_hat = rope(rms(q) w_q), k_hat = rope(rms(k) w_k) per head, both
//                      stored bf16 (k_hat into the caller's K cache), v copied to the V cache;
//   flash_attn_kernel  causal softmax attention, GQA, on the tensor cores, with the output
//                      gate o * sigmoid(g) in its epilogue.
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
// One warp per (token, head): lane l holds dims 8l .. 8l+7 (16-byte loads); the rotary
// pairs (i, i + 32) of dims 0 .. 63 sit in lanes l and l ^ 4 (l < 8).  The angles are
// formed and reduced modulo 2 pi in fp64 (positions reach 262,144), then sincosf.
constexpr int kQkThreads = 256;
constexpr int kDevErrCacheFull = 16;  // a sequence's KV cache has no row for its new token

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
};

__global__ void __launch_bounds__(kQkThreads) attn_qk_kernel(AttnQkParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * (kQkThreads / 32) + warp;  // (token, head)
  constexpr int kHeads = kAHq + kAHkv + kAHkv;  // q heads, k heads, v heads
  if (item >= p.T_tot * kHeads) return;
  const long long t = item / kHeads;
  const int hh = static_cast<int>(item % kHeads);
  const long long n = t / p.T;
  const long long pos = (p.pos_base ? p.pos_base[n] : 0) + t % p.T;
  if (pos >= p.cap) {  // no room in the cache: nothing is written for this sequence
    if (lane == 0 && hh == 0 && p.err) atomicOr(p.err, kDevErrCacheFull);
    return;
  }
  const long long crow = n * p.cap + pos;  // cache row of this token
  const bf16* row = p.proj + t * p.ld_p;
  if (hh >= kAHq + kAHkv) {  // v: a copy into the cache
    const int h = hh - kAHq - kAHkv;
    const uint4 u = reinterpret_cast<const uint4*>(row + 2 * kAHq * kAD + kAHkv * kAD + h * kAD)[lane];
    reinterpret_cast<uint4*>(p.v_cache + (crow * kAHkv + h) * kAD)[lane] = u;
    return;
  }
  const bool is_q = hh < kAHq;
  const int h = is_q ? hh : hh - kAHq;
  const bf16* src = is_q ? row + h * kAD : row + 2 * kAHq * kAD + h * kAD;
  float x[8], w[8];
  unpack8f(reinterpret_cast<const uint4*>(src)[lane], x);
  unpack8f(reinterpret_cast<const uint4*>(is_q ? p.q_norm_w : p.k_norm_w)[lane], w);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss * (1.0f / kAD) + 1e-6f);
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = x[e] * inv * w[e];
  // rotary on dims 0 .. 63 (lanes 0 .. 7): lane l < 4 holds x1 = dims 8l.., lane l + 4 holds x2
  float partner[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) partner[e] = __shfl_xor_sync(0xffffffffu, x[e], 4);
  if (lane < 8) {
    const double posd = static_cast<double>(pos);
    const int i0 = 8 * (lane & 3);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double theta = exp(-static_cast<double>(i0 + e) / (kARope / 2) * log(kARopeBase));
      const double ang = fmod(posd * theta, 6.283185307179586476925286766559);
      float sn, cs;
      sincosf(static_cast<float>(ang), &sn, &cs);
      // x1' = x1 c - x2 s (lanes 0..3), x2' = x2 c + x1 s (lanes 4..7)
      x[e] = lane < 4 ? fmaf(x[e], cs, -partner[e] * sn) : fmaf(x[e], cs, partner[e] * sn);
    }
  }
  bf16* dst = is_q ? p.q_hat + (t * kAHq + h) * kAD : p.k_cache + (crow * kAHkv + h) * kAD;
  reinterpret_cast<uint4*>(dst)[lane] = pack8f(x);
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
// head, sequence) takes up to kDecSplit cache rows and the KV head's 6 query heads, in fp32:
// pass 1 scores (warp = token, lane = 8 dims, a reduction over the lanes per head), per-head
// max and exponentials, pass 2 the weighted V sum (lane = 8 dims of the 6 heads), partials
// (o, m, l) to scratch.  attn_decode_combine_kernel merges the splits per (sequence, query
// head), applies 1/l and sigmoid(g), writes bf16; a last small kernel advances cache_len.  The cache is read
// once per KV head per step: HBM-bound by design.
constexpr int kDecSplit = 256;
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

__global__ void __launch_bounds__(kDecThreads, 3) attn_decode_kernel(AttnDecParams p) {
  const int sp = blockIdx.x, kvh = blockIdx.y, n = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float qs[kAGrp][kAD];
  __shared__ float sc[kAGrp][kDecSplit];
  __shared__ float os[kAGrp][kAD];
  __shared__ float mh[kAGrp], lh[kAGrp];
  float* part = p.part + ((static_cast<long long>(n) * kAHkv + kvh) * p.n_splits + sp) * kAGrp * kDecPart;
  const int len = p.cache_len[n] + 1;
  const int t0 = sp * kDecSplit, t1 = min(t0 + kDecSplit, len);
  if (len > p.cap || t0 >= t1) {  // nothing here (or no room in the cache): an empty partial
    if (threadIdx.x < kAGrp) {
      part[threadIdx.x * kDecPart + kAD] = -INFINITY;
      part[threadIdx.x * kDecPart + kAD + 1] = 0.f;
    }
    return;
  }
  for (int x = threadIdx.x; x < kAGrp * kAD; x += kDecThreads) {
    const int j = x / kAD, d = x % kAD;
    qs[j][d] = __bfloat162float(p.q_hat[(static_cast<long long>(n) * kAHq + kvh * kAGrp + j) * kAD + d]) * 0.0625f;
  }
  for (int x = threadIdx.x; x < kAGrp * kAD; x += kDecThreads) os[x / kAD][x % kAD] = 0.f;
  __syncthreads();
  const bf16* kbase = p.k_cache + (static_cast<long long>(n) * p.cap * kAHkv + kvh) * kAD;
  const bf16* vbase = p.v_cache + (static_cast<long long>(n) * p.cap * kAHkv + kvh) * kAD;
  // pass 1: scores (already scaled by 1/sqrt(256) through q).  Lane = 8 dims; four tokens per
  // step with their loads issued together; the 6 per-lane partial dot products (padded to 8)
  // are summed over the 32 lanes by a transposed butterfly: at each of the first three steps a
  // lane keeps half of its values and hands the other half to its partner, so lane l ends with
  // the full sum of value (l >> 2) & 7 after 9 shuffles instead of 30.
  float qr[kAGrp][8];
#pragma unroll
  for (int j = 0; j < kAGrp; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) qr[j][e] = qs[j][8 * lane + e];
  const int b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
  for (int tb = t0 + 4 * warp; tb < t1; tb += 4 * (kDecThreads / 32)) {
    uint4 kr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      kr[u] = tb + u < t1 ? reinterpret_cast<const uint4*>(kbase + static_cast<long long>(tb + u) * kAHkv * kAD)[lane]
                          : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float kf[8];
      unpack8f(kr[u], kf);
      float v8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float a = 0.f;
        if (j < kAGrp) {
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qr[j][e], kf[e], a);
        }
        v8[j] = a;
      }
      // step 1 (lanes l, l ^ 16): keep values 4 b4 .. 4 b4 + 3
      float v4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float keep = b4 ? v8[i + 4] : v8[i], give = b4 ? v8[i] : v8[i + 4];
        v4[i] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
      }
      // step 2 (l ^ 8): keep 2 b3 .. 2 b3 + 1 of those
      float v2[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float keep = b3 ? v4[i + 2] : v4[i], give = b3 ? v4[i] : v4[i + 2];
        v2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
      }
      // step 3 (l ^ 4): keep b2
      const float keep = b2 ? v2[1] : v2[0], give = b2 ? v2[0] : v2[1];
      float v1 = keep + __shfl_xor_sync(0xffffffffu, give, 4);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
      const int head = 4 * b4 + 2 * b3 + b2;
      if ((lane & 3) == 0 && head < kAGrp && tb + u < t1) sc[head][tb + u - t0] = v1;
    }
  }
  __syncthreads();
  // per-head max, exponentials and sum (warp j < 6 takes head j)
  if (warp < kAGrp) {
    float m = -INFINITY;
    for (int i = lane; i < t1 - t0; i += 32) m = fmaxf(m, sc[warp][i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int i = lane; i < t1 - t0; i += 32) {
      const float e = expf(sc[warp][i] - m);
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
  // pass 2: o[j] = sum_t p[j][t] v[t], four tokens per step with their loads issued together
  float acc[kAGrp][8];
#pragma unroll
  for (int j = 0; j < kAGrp; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
  for (int tb = t0 + 4 * warp; tb < t1; tb += 4 * (kDecThreads / 32)) {
    uint4 vr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      vr[u] = tb + u < t1 ? reinterpret_cast<const uint4*>(vbase + static_cast<long long>(tb + u) * kAHkv * kAD)[lane]
                          : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (tb + u >= t1) break;
      float vf[8];
      unpack8f(vr[u], vf);
#pragma unroll
      for (int j = 0; j < kAGrp; ++j) {
        const float pj = sc[j][tb + u - t0];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[j][e] = fmaf(pj, vf[e], acc[j][e]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kAGrp; ++j)
#pragma unroll
    for (int e = 0; e < 8; ++e) atomicAdd(&os[j][8 * lane + e], acc[j][e]);
  __syncthreads();
  for (int x = threadIdx.x; x < kAGrp * kAD; x += kDecThreads) part[(x / kAD) * kDecPart + x % kAD] = os[x / kAD][x % kAD];
  if (threadIdx.x < kAGrp) {
    part[threadIdx.x * kDecPart + kAD] = mh[threadIdx.x];
    part[threadIdx.x * kDecPart + kAD + 1] = lh[threadIdx.x];
  }
}

// merge the splits of (sequence n, query head h): o = sum_s o_s e^{m_s - M} / sum_s l_s e^{m_s - M}
__global__ void __launch_bounds__(kAD) attn_decode_combine_kernel(AttnDecParams p, const bf16* g, long long ld_g,
                                                                  bf16* out) {
  const int n = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  const int kvh = h / kAGrp, j = h % kAGrp;
  const int len = p.cache_len[n] + 1;
  if (len > p.cap) {  // reported by the cache write; nothing was attended: a zero output row
    out[(static_cast<long long>(n) * kAHq + h) * kAD + d] = __float2bfloat16(0.f);
    return;
  }
  const int used = (len + kDecSplit - 1) / kDecSplit;
  const float* base = p.part + (static_cast<long long>(n) * kAHkv + kvh) * p.n_splits * kAGrp * kDecPart;
  float M = -INFINITY;
  for (int s2 = 0; s2 < used; ++s2) M = fmaxf(M, base[(s2 * kAGrp + j) * kDecPart + kAD]);
  float L = 0.f, O = 0.f;
  for (int s2 = 0; s2 < used; ++s2) {
    const float* ps = base + (s2 * kAGrp + j) * kDecPart;
    const float w = expf(ps[kAD] - M);
    L = fmaf(ps[kAD + 1], w, L);
    O = fmaf(ps[d], w, O);
  }
  const float gv = __bfloat162float(g[static_cast<long long>(n) * ld_g + h * kAD + d]);
  out[(static_cast<long long>(n) * kAHq + h) * kAD + d] = __float2bfloat16(O / L / (1.0f + expf(-gv)));
}

// the step is complete: each sequence's cache holds one more row (unless it was full)
__global__ void attn_cache_advance_kernel(int* cache_len, int N, int cap) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N && cache_len[n] < cap) cache_len[n] += 1;
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
  const long long items = T_tot * (kAHq + 2 * kAHkv);
  attn_qk_kernel<<<static_cast<unsigned>((items + kQkThreads / 32 - 1) / (kQkThreads / 32)), kQkThreads, 0,
                   stream>>>(qp);
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
