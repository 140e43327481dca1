// Single-token decode step of the gated-delta-rule mixer.
//
// Agnes-3.0-Flash model card, "Architecture" table, row "Delta-rule layers":
// causal conv (kernel 4) in front, gated RMS-norm after, fp32 recurrent state;
// "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model", section
// "Feed-Forward and Positional Encoding", paragraph on the Gated Delta Rule:
// erase the key's old association, then write, under a forget gate.  Per value head and state row
// r (d_v index) the step reads the row once and writes it once:
//   sk = s_r . k, sq = s_r . q,  delta = beta (v_r - alpha sk),
//   s_r <- alpha s_r + delta k,   o_r = alpha sq + delta (k . q),
// which is S_t = alpha S_{t-1}(I - beta k k^T) + beta v k^T, o = S_t q.
//
// One CTA per (sequence, key head): it owns the key head's q/k conv channels
// and the value channels and state rows of the key head's value heads, so the
// conv state and the recurrent state are updated in place without races.
#include "gdn_kernels.cuh"

namespace gdn {

namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerIter = 8;  // state rows in flight per warp

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__global__ void __launch_bounds__(kDecThreads) gdn_decode_kernel(DecodeParams p) {
  const int kh = blockIdx.x, n = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H_k = p.H_k, H_v = p.H_v, G = H_v / H_k;
  const long long C_conv = static_cast<long long>(2 * H_k + H_v) * kD;

  extern __shared__ float dsm[];
  float* feat = dsm;                     // (2 + G) * 128 post-conv features: q | k | v(G heads)
  float* o_s = feat + (2 + G) * kD;      // G * 128 pre-norm outputs
  __shared__ float red[4];
  __shared__ float alpha_s[8], beta_s[8];

  // ---- conv front end for this token; shift the conv state in place
  const int n_ch = (2 + G) * kD;
  bf16* cs = p.conv_state + static_cast<long long>(n) * 3 * C_conv;
  for (int j = tid; j < n_ch; j += kDecThreads) {
    long long c;
    float x;
    if (j < kD) {
      c = static_cast<long long>(kh) * kD + j;
      x = __bfloat162float(p.q[n * p.sq + kh * kD + j]);
    } else if (j < 2 * kD) {
      c = static_cast<long long>(H_k) * kD + kh * kD + (j - kD);
      x = __bfloat162float(p.k[n * p.sk + kh * kD + (j - kD)]);
    } else {
      const int vj = j - 2 * kD;  // 0 .. G*128
      c = static_cast<long long>(2 * H_k) * kD + static_cast<long long>(kh) * G * kD + vj;
      x = __bfloat162float(p.v[n * p.sv + static_cast<long long>(kh) * G * kD + vj]);
    }
    const float h0 = __bfloat162float(cs[c]);
    const float h1 = __bfloat162float(cs[C_conv + c]);
    const float h2 = __bfloat162float(cs[2 * C_conv + c]);
    const bf16* w = p.conv_w + c * kTaps;
    float y = __bfloat162float(w[0]) * h0;
    y = fmaf(__bfloat162float(w[1]), h1, y);
    y = fmaf(__bfloat162float(w[2]), h2, y);
    y = fmaf(__bfloat162float(w[3]), x, y);
    feat[j] = silu_f(y);
    cs[c] = __float2bfloat16(h1);
    cs[C_conv + c] = __float2bfloat16(h2);
    cs[2 * C_conv + c] = __float2bfloat16(x);
  }
  if (tid < G) {
    const int h = kh * G + tid;
    const float a = __bfloat162float(p.a[n * p.sa + h]);
    const float b = __bfloat162float(p.b[n * p.sb + h]);
    alpha_s[tid] = expf(-expf(p.A_log[h]) * softplus_f(a));
    beta_s[tid] = sigmoid_f(b);
  }
  __syncthreads();
  // L2 norms of q (warp 0) and k (warp 1)
  if (warp < 2) {
    float ss = 0.f;
    for (int j = lane; j < kD; j += 32) {
      const float x = feat[warp * kD + j];
      ss = fmaf(x, x, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = rsqrtf(ss + 1e-6f);
  }
  __syncthreads();
  // normalised q, k slices of this lane (d_k elements 4*lane .. 4*lane+3)
  float qv[4], kv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    qv[e] = feat[4 * lane + e] * red[0] * p.scale;
    kv[e] = feat[kD + 4 * lane + e] * red[1];
  }
  const float kq = warp_sum(qv[0] * kv[0] + qv[1] * kv[1] + qv[2] * kv[2] + qv[3] * kv[3]);

  // ---- stream the state rows: rows r = head j * 128 + d_v index
  const int n_rows = G * kD;
  float* S = p.state + (static_cast<long long>(n) * H_v + static_cast<long long>(kh) * G) * kD * kD;
  for (int r0 = warp * kRowsPerIter; r0 < n_rows; r0 += (kDecThreads / 32) * kRowsPerIter) {
    float4 s[kRowsPerIter];
#pragma unroll
    for (int u = 0; u < kRowsPerIter; ++u)
      s[u] = __ldcs(reinterpret_cast<const float4*>(S + static_cast<long long>(r0 + u) * kD) + lane);
#pragma unroll
    for (int u = 0; u < kRowsPerIter; ++u) {
      const int r = r0 + u, j = r >> 7;
      float sk = s[u].x * kv[0] + s[u].y * kv[1] + s[u].z * kv[2] + s[u].w * kv[3];
      float sq = s[u].x * qv[0] + s[u].y * qv[1] + s[u].z * qv[2] + s[u].w * qv[3];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sk += __shfl_xor_sync(0xffffffffu, sk, o);
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
      }
      const float al = alpha_s[j], be = beta_s[j];
      const float delta = be * (feat[2 * kD + r] - al * sk);
      float4 ns;
      ns.x = fmaf(al, s[u].x, delta * kv[0]);
      ns.y = fmaf(al, s[u].y, delta * kv[1]);
      ns.z = fmaf(al, s[u].z, delta * kv[2]);
      ns.w = fmaf(al, s[u].w, delta * kv[3]);
      __stcs(reinterpret_cast<float4*>(S + static_cast<long long>(r) * kD) + lane, ns);
      if (lane == 0) o_s[r] = fmaf(al, sq, delta * kq);
    }
  }
  __syncthreads();

  // ---- gated RMS-norm per value head (warp j handles head j)
  for (int j = warp; j < G; j += kDecThreads / 32) {
    const int h = kh * G + j;
    float ss = 0.f;
    for (int d = lane; d < kD; d += 32) ss = fmaf(o_s[j * kD + d], o_s[j * kD + d], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss * (1.0f / kD) + 1e-6f);
    for (int d = lane; d < kD; d += 32) {
      const float z = __bfloat162float(p.z[n * p.sz + static_cast<long long>(h) * kD + d]);
      const float y = o_s[j * kD + d] * inv * __bfloat162float(p.norm_w[d]) * silu_f(z);
      p.out[(static_cast<long long>(n) * H_v + h) * kD + d] = __float2bfloat16(y);
    }
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream, void* const* events) {
  const int G = p.H_v / p.H_k;
  const size_t smem = static_cast<size_t>((2 + G) * kD + G * kD) * sizeof(float);
  dim3 grid(p.H_k, p.N);
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[0]), stream);
  gdn_decode_kernel<<<grid, kDecThreads, smem, stream>>>(p);
  cudaError_t err = cudaGetLastError();
  if (events) cudaEventRecord(static_cast<cudaEvent_t>(events[1]), stream);
  return err;
}

}  // namespace gdn
