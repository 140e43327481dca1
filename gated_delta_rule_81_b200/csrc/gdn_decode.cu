// Decode steps of the gated-delta-rule mixer: T = 1 .. 8 new tokens per sequence.
//
// Agnes-3.0-Flash model card, "Architecture" table, row "Delta-rule layers":
// causal conv (kernel 4) in front, gated RMS-norm after, fp32 recurrent state;
// "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model", section
// "Feed-Forward and Positional Encoding", paragraph on the Gated Delta Rule:
// erase the key's old association, then write, under a forget gate.  Per value
// head, state row r (d_v index) and new token t, in token order:
//   sk = s_r . k_t, sq = s_r . q_t,  delta = beta_t (v_{t,r} - alpha_t sk),
//   s_r <- alpha_t s_r + delta k_t,   o_{t,r} = alpha_t sq + delta (k_t . q_t),
// which is S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
// A state row is read from HBM once and written once per call whatever T is: the
// T updates run on the row in registers, so the call's HBM traffic is one state
// round trip for T tokens.
//
// One CTA per (sequence, key head), or, when that grid would leave SMs idle (few
// sequences), one CTA per (sequence, value head) with the G CTAs of a key head in one
// thread-block cluster.  A CTA owns the state rows and value channels of its value heads,
// so the recurrent state and the v part of the conv state are updated in place without
// races; the q/k conv channels of a key head are read by every CTA of its cluster and
// written by the cluster's first CTA after a cluster barrier, i.e. after all of them
// have read the history.  Each CTA of a cluster normalises q and k itself (the same code
// on the same data), so both grids give bitwise equal results.
// Every token goes through the same code whatever T is, so T calls with one token
// and one call with T tokens give bitwise equal results.
//
// Latency: everything the CTA reads besides the state (the T raw q/k/v rows, the
// conv history and taps, z) is staged into shared memory by one burst of 16-byte
// asynchronous copies, so the front end waits on global memory once; each warp asks
// L2 for its next block of state rows before it works on the current one.
#include "gdn_kernels.cuh"

namespace gdn {

namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerIter = 16;  // state rows per warp and block (8 KiB, contiguous)
constexpr int kRowBlockBytes = kRowsPerIter * kD * 4;

// Shared-memory float4 load kept where it is written (not merged with an earlier load of
// the same address), so the k slice is read again for the update rather than held in
// registers across the reduction.
__device__ __forceinline__ float4 lds4_again(const float4* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
  return v;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Dynamic shared memory, in bytes, for T tokens and G value heads per key head (n_ch = (2 + G) 128):
//   feat  f32 [T][n_ch]        post-conv q | k | v, then q, k normalised in place
//   raw   staging              bf16 x [T][n_ch] | bf16 conv history [3][n_ch] | bf16 conv taps [n_ch][4];
//                              after the conv it holds the f32 pre-norm outputs [T][G 128]
//   z     bf16 [T][G][128]
struct DecodeSmem {
  int feat, raw, hist, taps, z, total;
};

__host__ __device__ inline DecodeSmem decode_smem(int T, int G) {
  const int n_ch = (2 + G) * kD;
  DecodeSmem L;
  L.feat = 0;
  L.raw = T * n_ch * 4;
  L.hist = L.raw + T * n_ch * 2;
  L.taps = L.hist + 3 * n_ch * 2;
  const int raw_end = L.taps + n_ch * kTaps * 2;
  const int o_end = L.raw + T * G * kD * 4;
  L.z = raw_end > o_end ? raw_end : o_end;
  L.total = L.z + T * G * kD * 2;
  return L;
}

// global channel of CTA channel j: q head kh, k head kh, then the CTA's value heads from hv0 on
__device__ __forceinline__ long long conv_channel(int j, int kh, int H_k, int hv0) {
  return j < kD       ? static_cast<long long>(kh) * kD + j
         : j < 2 * kD ? static_cast<long long>(H_k + kh) * kD + (j - kD)
                      : static_cast<long long>(2 * H_k + hv0) * kD + (j - 2 * kD);
}

// every thread of the cluster arrives, then waits for all the others (release / acquire)
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kDecThreads, 2) gdn_decode_kernel(DecodeParams p) {
  // grid (parts, H_k, N): a part takes G / parts consecutive value heads of key head kh
  const int part = blockIdx.x, parts = gridDim.x, kh = blockIdx.y, n = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H_k = p.H_k, H_v = p.H_v, G = H_v / H_k / parts, T = p.T;
  const int hv0 = (kh * parts + part) * G;  // the CTA's first value head; G = its value heads
  const long long C_conv = static_cast<long long>(2 * H_k + H_v) * kD;
  const int slot = p.state_slot ? p.state_slot[n] : n;
  if (slot < 0 || slot >= p.n_slots) {  // the same value in every thread: the CTA leaves together
    if (tid == 0 && p.err) atomicOr(p.err, kDevErrBadSlot);
    return;
  }
  const int n_ch = (2 + G) * kD, n_rows = G * kD;
  float* S = p.state + (static_cast<long long>(slot) * H_v + hv0) * kD * kD;
  // the first block of state rows of each warp starts on its way to L2 now
  if (lane == 0) prefetch_l2(S + static_cast<long long>(warp) * kRowsPerIter * kD, kRowBlockBytes);

  extern __shared__ __align__(16) unsigned char dsm_raw[];
  const DecodeSmem L = decode_smem(T, G);
  float* feat = reinterpret_cast<float*>(dsm_raw + L.feat);
  bf16* xraw = reinterpret_cast<bf16*>(dsm_raw + L.raw);
  bf16* hist = reinterpret_cast<bf16*>(dsm_raw + L.hist);
  bf16* taps = reinterpret_cast<bf16*>(dsm_raw + L.taps);
  float* o_s = reinterpret_cast<float*>(dsm_raw + L.raw);  // reuses the staging area after the conv
  bf16* z_s = reinterpret_cast<bf16*>(dsm_raw + L.z);
  __shared__ float red[kMaxDecodeTokens][2];
  __shared__ float kq_s[kMaxDecodeTokens];
  __shared__ float alpha_s[kMaxDecodeTokens * 8], beta_s[kMaxDecodeTokens * 8];
  __shared__ float normw_s[kD];

  // ---- stage the CTA's inputs with 16-byte copies (8 bf16 each; segments of 128 channels
  // are 16-byte aligned because every pointer and stride is)
  const int n_p16 = n_ch / 8;  // 16-byte pieces of one row of the CTA's n_ch channels
  for (int i = tid; i < T * n_p16; i += kDecThreads) {  // raw q | k | v of the T tokens
    const int t = i / n_p16, e = (i % n_p16) * 8;
    const long long tok = static_cast<long long>(n) * T + t;
    const bf16* src = e < kD       ? p.q + tok * p.sq + static_cast<long long>(kh) * kD + e
                      : e < 2 * kD ? p.k + tok * p.sk + static_cast<long long>(kh) * kD + (e - kD)
                                   : p.v + tok * p.sv + static_cast<long long>(hv0) * kD + (e - 2 * kD);
    cp_async16(xraw + t * n_ch + e, src);
  }
  const bf16* cs_in = p.conv_state + static_cast<long long>(slot) * 3 * C_conv;
  for (int i = tid; i < 3 * n_p16; i += kDecThreads) {  // conv history rows
    const int row = i / n_p16, e = (i % n_p16) * 8;
    cp_async16(hist + row * n_ch + e, cs_in + row * C_conv + conv_channel(e, kh, H_k, hv0));
  }
  for (int i = tid; i < n_ch / 2; i += kDecThreads) {  // conv taps: one piece = 2 channels x 4 taps
    const int e = 2 * i;
    cp_async16(taps + e * kTaps, p.conv_w + conv_channel(e, kh, H_k, hv0) * kTaps);
  }
  for (int i = tid; i < T * G * (kD / 8); i += kDecThreads) {  // z of the T tokens and G heads
    const int t = i / (G * (kD / 8)), rem = i % (G * (kD / 8)), jh = rem / (kD / 8), e = (rem % (kD / 8)) * 8;
    const long long tok = static_cast<long long>(n) * T + t;
    cp_async16(z_s + (t * G + jh) * kD + e, p.z + tok * p.sz + static_cast<long long>(hv0 + jh) * kD + e);
  }
  cp_async_commit();
  for (int x = tid; x < T * G; x += kDecThreads) {  // gates (a and b are only 2-byte aligned)
    const int t = x / G, jh = x % G, h = hv0 + jh;
    const long long tok = static_cast<long long>(n) * T + t;
    const float a = __bfloat162float(p.a[tok * p.sa + h]);
    const float b = __bfloat162float(p.b[tok * p.sb + h]);
    alpha_s[t * 8 + jh] = expf(-expf(p.A_log[h]) * softplus_f(a));
    beta_s[t * 8 + jh] = sigmoid_f(b);
  }
  if (tid < kD) normw_s[tid] = __bfloat162float(p.norm_w[tid]);
  cp_async_wait_all();
  __syncthreads();
  if (parts > 1) cluster_barrier();  // every CTA of the key head holds the old q/k history now

  // ---- causal conv over the T new tokens (a sliding window over the 3 history rows);
  // the conv state takes the last three raw tokens
  bf16* cs_out = p.conv_state + static_cast<long long>(slot) * 3 * C_conv;
  for (int j = tid; j < n_ch; j += kDecThreads) {
    float h0 = __bfloat162float(hist[j]);
    float h1 = __bfloat162float(hist[n_ch + j]);
    float h2 = __bfloat162float(hist[2 * n_ch + j]);
    const bf16* w = taps + j * kTaps;
    const float w0 = __bfloat162float(w[0]), w1 = __bfloat162float(w[1]), w2 = __bfloat162float(w[2]),
                w3 = __bfloat162float(w[3]);
    for (int t = 0; t < T; ++t) {
      const float x = __bfloat162float(xraw[t * n_ch + j]);
      float y = w0 * h0;
      y = fmaf(w1, h1, y);
      y = fmaf(w2, h2, y);
      y = fmaf(w3, x, y);
      feat[t * n_ch + j] = silu_f(y);
      h0 = h1;
      h1 = h2;
      h2 = x;
    }
    if (part == 0 || j >= 2 * kD) {  // q/k channels: the cluster's first CTA alone
      const long long c = conv_channel(j, kh, H_k, hv0);
      cs_out[c] = __float2bfloat16(h0);
      cs_out[C_conv + c] = __float2bfloat16(h1);
      cs_out[2 * C_conv + c] = __float2bfloat16(h2);
    }
  }
  __syncthreads();
  // L2 norms of q and k of every token (item = 2 t + which)
  for (int item = warp; item < 2 * T; item += kDecThreads / 32) {
    const int t = item >> 1, which = item & 1;
    float ss = 0.f;
    for (int j = lane; j < kD; j += 32) {
      const float x = feat[t * n_ch + which * kD + j];
      ss = fmaf(x, x, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[t][which] = rsqrtf(ss + 1e-6f);
  }
  __syncthreads();
  // normalised q (times scale) and k in place; k . q per token
  for (int x = tid; x < T * 2 * kD; x += kDecThreads) {
    const int t = x / (2 * kD), j = x % (2 * kD);
    const float f = feat[t * n_ch + j] * red[t][j >> 7];
    feat[t * n_ch + j] = j < kD ? f * p.scale : f;
  }
  __syncthreads();
  for (int t = warp; t < T; t += kDecThreads / 32) {
    const float4 qv = reinterpret_cast<const float4*>(feat + t * n_ch)[lane];
    const float4 kv = reinterpret_cast<const float4*>(feat + t * n_ch + kD)[lane];
    const float kq = warp_sum(qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w);
    if (lane == 0) kq_s[t] = kq;
  }
  __syncthreads();

  // ---- stream the state rows (r = value head j * 128 + d_v index): read once, T updates, write once.
  // A warp takes 16 contiguous rows at a time.  Eight lanes share a row (lane = 8 g + c): lane c
  // holds the float4 columns c + 8 m (m = 0 .. 3) of rows r0 + g + 4 u (u = 0 .. 3), so each
  // q / k slice read from shared memory serves four rows and the update needs no exchange.
  // The eight partial dot products of a lane (s.k, s.q of its four rows) are summed over the
  // eight lanes of the row group by a transposed butterfly: at each step a lane keeps half of
  // its values and hands the other half to its partner, so lane c ends with the complete
  // s.k, s.q of row u = c >> 1 after 8 shuffles (a plain butterfly on all 8 values takes 24).
  const int g = lane >> 3, c = lane & 7;
  const bool b2 = (c >> 2) & 1, b1 = (c >> 1) & 1;
  const int u_me = c >> 1;
  for (int r0 = warp * kRowsPerIter; r0 < n_rows; r0 += (kDecThreads / 32) * kRowsPerIter) {
    const int jh = r0 >> 7;  // the 16 rows belong to one value head
    float4 s[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int m = 0; m < 4; ++m)
        s[u][m] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<long long>(r0 + g + 4 * u) * kD) + c + 8 * m);
    const int r_next = r0 + (kDecThreads / 32) * kRowsPerIter;
    if (lane == 0 && r_next < n_rows) prefetch_l2(S + static_cast<long long>(r_next) * kD, kRowBlockBytes);
    for (int t = 0; t < T; ++t) {
      const float4* qt = reinterpret_cast<const float4*>(feat + t * n_ch);
      const float4* kt = qt + kD / 4;
      float2 ak[4], aq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) ak[u] = aq[u] = make_float2(0.f, 0.f);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 kk = kt[c + 8 * m];
        const float4 qq = qt[c + 8 * m];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 s01 = make_float2(s[u][m].x, s[u][m].y), s23 = make_float2(s[u][m].z, s[u][m].w);
          ak[u] = __ffma2_rn(s01, make_float2(kk.x, kk.y), ak[u]);
          ak[u] = __ffma2_rn(s23, make_float2(kk.z, kk.w), ak[u]);
          aq[u] = __ffma2_rn(s01, make_float2(qq.x, qq.y), aq[u]);
          aq[u] = __ffma2_rn(s23, make_float2(qq.z, qq.w), aq[u]);
        }
      }
      // (s.k, s.q) partial sums of the lane's four rows
      float2 d[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) d[u] = __fadd2_rn(make_float2(ak[u].x, aq[u].x), make_float2(ak[u].y, aq[u].y));
      // step 1 (lanes c, c ^ 4): keep rows 2 b2 + {0, 1}
      float2 e[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 keep = b2 ? d[i + 2] : d[i], give = b2 ? d[i] : d[i + 2];
        const float2 got = make_float2(__shfl_xor_sync(0xffffffffu, give.x, 4),
                                       __shfl_xor_sync(0xffffffffu, give.y, 4));
        e[i] = __fadd2_rn(keep, got);
      }
      // step 2 (lanes c, c ^ 2): keep row 2 b2 + b1
      float2 f;
      {
        const float2 keep = b1 ? e[1] : e[0], give = b1 ? e[0] : e[1];
        const float2 got = make_float2(__shfl_xor_sync(0xffffffffu, give.x, 2),
                                       __shfl_xor_sync(0xffffffffu, give.y, 2));
        f = __fadd2_rn(keep, got);
      }
      // step 3 (lanes c, c ^ 1): both lanes complete row u_me
      f = __fadd2_rn(f, make_float2(__shfl_xor_sync(0xffffffffu, f.x, 1), __shfl_xor_sync(0xffffffffu, f.y, 1)));
      const float al = alpha_s[t * 8 + jh], be = beta_s[t * 8 + jh];
      const int r_me = r0 + g + 4 * u_me;
      const float delta_me = be * (feat[t * n_ch + 2 * kD + r_me] - al * f.x);
      if ((c & 1) == 0) o_s[t * n_rows + r_me] = fmaf(al, f.y, delta_me * kq_s[t]);
      const float2 al2 = make_float2(al, al);
      float2 d2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float delta = __shfl_sync(0xffffffffu, delta_me, (lane & ~7) + 2 * u);
        d2[u] = make_float2(delta, delta);
      }
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 kk = lds4_again(kt + c + 8 * m);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 lo = __ffma2_rn(al2, make_float2(s[u][m].x, s[u][m].y),
                                       __fmul2_rn(d2[u], make_float2(kk.x, kk.y)));
          const float2 hi = __ffma2_rn(al2, make_float2(s[u][m].z, s[u][m].w),
                                       __fmul2_rn(d2[u], make_float2(kk.z, kk.w)));
          s[u][m] = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int m = 0; m < 4; ++m)
        __stcs(reinterpret_cast<float4*>(S + static_cast<long long>(r0 + g + 4 * u) * kD) + c + 8 * m, s[u][m]);
  }
  __syncthreads();

  // ---- gated RMS-norm per (token, value head): one warp per pair
  for (int pr = warp; pr < T * G; pr += kDecThreads / 32) {
    const int t = pr / G, jh = pr % G, h = hv0 + jh;
    const long long tok = static_cast<long long>(n) * T + t;
    const float* ot = o_s + t * n_rows + jh * kD;
    const bf16* zt = z_s + (t * G + jh) * kD;
    float ss = 0.f;
    for (int dd = lane; dd < kD; dd += 32) ss = fmaf(ot[dd], ot[dd], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss * (1.0f / kD) + 1e-6f);
    for (int dd = lane; dd < kD; dd += 32) {
      const float y = ot[dd] * inv * normw_s[dd] * silu_f(__bfloat162float(zt[dd]));
      p.out[(tok * H_v + h) * kD + dd] = __float2bfloat16(y);
    }
  }
}

}  // namespace

// CTAs per key head: G (one per value head, a cluster of G <= 8) while one CTA per
// (sequence, key head) would leave SMs idle, else 1.
int decode_parts(const DecodeParams& p) {
  const int G = p.H_v / p.H_k;
  if (G == 1) return 1;
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 1;
  return static_cast<long long>(p.N) * p.H_k < n_sm ? G : 1;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream, void* const* events) {
  const int parts = decode_parts(p);
  const int smem = decode_smem(p.T, p.H_v / p.H_k / parts).total;
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(gdn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(parts, p.H_k, p.N);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = parts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = parts > 1 ? 1 : 0;
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[0]), stream);
  cudaError_t err = cudaLaunchKernelEx(&cfg, gdn_decode_kernel, p);
  if (err == cudaSuccess) err = cudaGetLastError();
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), stream);
  return err;
}

}  // namespace gdn
