// C ABI of the gated-delta-rule mixer: argument validation, workspace layout
// and kernel launches.  Declared in include/gdn.h.
#include <limits.h>
#include <stdint.h>
#include <stdlib.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/gdn.h"
#include "gdn_kernels.cuh"

using gdn::bf16;

namespace {

// NVTX ranges named after the entry points, when GDN_NVTX is set (to anything but 0) in the
// environment; read once.  NVTX3 is header-only and loads nothing unless a profiler injects it.
bool nvtx_on() {
  static const bool on = [] {
    const char* e = getenv("GDN_NVTX");
    return e && *e && !(e[0] == '0' && e[1] == 0);
  }();
  return on;
}

struct NvtxRange {
  bool on;
  explicit NvtxRange(const char* name) : on(nvtx_on()) {
    if (on) nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

// leading dimension of the layer's projection buffer: n_in rounded up to 8 (16-byte rows)
long long layer_ld_proj(int H_k, int H_v) {
  return (2LL * H_k * GDN_HEAD_DIM + 2LL * H_v * GDN_HEAD_DIM + 2LL * H_v + 7) / 8 * 8;
}

// chunk_base[N+1] and seq_order[N] (ints) after the 1 KiB header
size_t chunk_base_bytes(int N) { return round_up(sizeof(int) * (2 * static_cast<size_t>(N) + 1), 1024); }

// Common checks of the per-token inputs; T_tot tokens.
gdn_status check_inputs(const gdn_inputs* in, long long T_tot) {
  if (!in) return GDN_ERR_INVALID_ARG;
  if (in->H_k <= 0 || in->H_v <= 0 || in->H_v % in->H_k != 0) return GDN_ERR_INVALID_ARG;
  if (in->H_v / in->H_k > 8) return GDN_ERR_UNSUPPORTED;
  if (T_tot == 0) return GDN_OK;
  if (!in->q || !in->k || !in->v || !in->a || !in->b || !in->z || !in->conv_w || !in->A_log || !in->norm_w)
    return GDN_ERR_INVALID_ARG;
  const long long qk = static_cast<long long>(in->H_k) * GDN_HEAD_DIM, vz = static_cast<long long>(in->H_v) * GDN_HEAD_DIM;
  if (in->stride_q < qk || in->stride_k < qk || in->stride_v < vz || in->stride_z < vz || in->stride_a < in->H_v ||
      in->stride_b < in->H_v)
    return GDN_ERR_INVALID_ARG;
  if (!aligned16(in->q) || !aligned16(in->k) || !aligned16(in->v) || !aligned16(in->z) || !aligned16(in->conv_w))
    return GDN_ERR_MISALIGNED;
  if ((in->stride_q | in->stride_k | in->stride_v | in->stride_z) & 7) return GDN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(in->a) | reinterpret_cast<uintptr_t>(in->b) |
       reinterpret_cast<uintptr_t>(in->norm_w)) & 1u)
    return GDN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(in->A_log) & 3u) return GDN_ERR_MISALIGNED;
  return GDN_OK;
}

// `out` must not overlap any input read by the same call
// bytes from the first element of a [T_tot] x stride input to the end of its last row's `width` channels
size_t input_extent(long long T_tot, long long stride, long long width) {
  return sizeof(bf16) * (static_cast<size_t>(T_tot - 1) * static_cast<size_t>(stride) + static_cast<size_t>(width));
}

gdn_status check_out_alias(const gdn_inputs* in, long long T_tot, const void* out) {
  const size_t ob = static_cast<size_t>(T_tot) * in->H_v * GDN_HEAD_DIM * sizeof(bf16);
  const long long qk = static_cast<long long>(in->H_k) * GDN_HEAD_DIM, vz = static_cast<long long>(in->H_v) * GDN_HEAD_DIM;
  if (overlap(out, ob, in->q, input_extent(T_tot, in->stride_q, qk)) ||
      overlap(out, ob, in->k, input_extent(T_tot, in->stride_k, qk)) ||
      overlap(out, ob, in->v, input_extent(T_tot, in->stride_v, vz)) ||
      overlap(out, ob, in->z, input_extent(T_tot, in->stride_z, vz)) ||
      overlap(out, ob, in->a, input_extent(T_tot, in->stride_a, in->H_v)) ||
      overlap(out, ob, in->b, input_extent(T_tot, in->stride_b, in->H_v)))
    return GDN_ERR_ALIAS;
  return GDN_OK;
}

// The mixer's inputs as columns of the layer's projection buffer [T_tot][ld_p]:
// q | k | v | z | a | b, read through the row stride ld_p (no copy).
gdn_inputs layer_mixer_inputs(const gdn_layer* L, const bf16* proj, long long ld_p) {
  const long long HkD = static_cast<long long>(L->H_k) * GDN_HEAD_DIM;
  const long long d_v = static_cast<long long>(L->H_v) * GDN_HEAD_DIM;
  gdn_inputs in = {};
  in.q = proj;
  in.k = proj + HkD;
  in.v = proj + 2 * HkD;
  in.z = proj + 2 * HkD + d_v;
  in.a = proj + 2 * HkD + 2 * d_v;
  in.b = proj + 2 * HkD + 2 * d_v + L->H_v;
  in.stride_q = in.stride_k = in.stride_v = in.stride_z = in.stride_a = in.stride_b = ld_p;
  in.conv_w = L->conv_w;
  in.A_log = L->A_log;
  in.norm_w = L->norm_w;
  in.H_k = L->H_k;
  in.H_v = L->H_v;
  in.scale = L->scale;
  in.schedule = L->schedule;
  return in;
}

// The aliasing rule of every prefill entry point, in one place: among the state and conv
// buffers and the output (out_bytes of it; nullptr when the call has none), a buffer the call
// writes (state_out, conv_out, out) overlaps no other one, except that state_out may be
// exactly state_in (the state is updated in place, each row by the one CTA that reads it).
gdn_status check_state_aliases(int H_k, int H_v, int n, const float* state_in, const float* state_out,
                               const void* conv_in, const void* conv_out, const void* out, size_t out_bytes) {
  const size_t state_bytes = static_cast<size_t>(n) * H_v * GDN_HEAD_DIM * GDN_HEAD_DIM * sizeof(float);
  const size_t conv_bytes = static_cast<size_t>(n) * 3 * (2 * H_k + H_v) * GDN_HEAD_DIM * sizeof(bf16);
  struct Buf {
    const void* p;
    size_t bytes;
    bool written;
  };
  const Buf b[5] = {{state_in, state_bytes, false}, {state_out, state_bytes, true}, {conv_in, conv_bytes, false},
                    {conv_out, conv_bytes, true}, {out, out_bytes, true}};
  for (int i = 0; i < 5; ++i)
    for (int j = i + 1; j < 5; ++j) {
      if (!b[i].written && !b[j].written) continue;
      if (i == 0 && j == 1 && state_in == state_out) continue;
      if (overlap(b[i].p, b[i].bytes, b[j].p, b[j].bytes)) return GDN_ERR_ALIAS;
    }
  return GDN_OK;
}

// The layer entry points check the states the mixer will take before their first launch, so
// that a rejected call launches nothing: alignment, and the aliasing rules of the mixer calls.
gdn_status check_layer_states(int H_k, int H_v, int n, const float* state_in, const float* state_out,
                              const void* conv_in, const void* conv_out) {
  if (!aligned16(state_in) || !aligned16(state_out) || !aligned16(conv_in) || !aligned16(conv_out))
    return GDN_ERR_MISALIGNED;
  return check_state_aliases(H_k, H_v, n, state_in, state_out, conv_in, conv_out, nullptr, 0);
}

// None of the state and conv buffers of a layer call may lie in its workspace (the projection,
// the mixer output and the mixer's scratch are written there).
bool states_in_workspace(int H_k, int H_v, int n, const void* s0, const void* s1, const void* c0, const void* c1,
                         const void* ws, size_t ws_bytes) {
  const size_t state_bytes = static_cast<size_t>(n) * H_v * GDN_HEAD_DIM * GDN_HEAD_DIM * sizeof(float);
  const size_t conv_bytes = static_cast<size_t>(n) * 3 * (2 * H_k + H_v) * GDN_HEAD_DIM * sizeof(bf16);
  return overlap(s0, state_bytes, ws, ws_bytes) || overlap(s1, state_bytes, ws, ws_bytes) ||
         overlap(c0, conv_bytes, ws, ws_bytes) || overlap(c1, conv_bytes, ws, ws_bytes);
}

gdn_status prefill_common(const gdn_inputs* in, int N, long long T_tot, long long n_chunks, const int* cu,
                          int T_uniform, const float* state_in, float* state_out, const void* conv_in,
                          void* conv_out, void* out, void* workspace, size_t workspace_bytes, int* err,
                          void* stream) {
  gdn_status st = check_inputs(in, T_tot);
  if (st != GDN_OK) return st;
  if (N == 0) return GDN_OK;
  if (T_tot > 0 && !out) return GDN_ERR_INVALID_ARG;
  if (T_tot > 0 && (st = check_out_alias(in, T_tot, out)) != GDN_OK) return st;
  if (!aligned16(out) || !aligned16(state_in) || !aligned16(state_out) || !aligned16(conv_in) ||
      !aligned16(conv_out) || !aligned16(workspace))
    return GDN_ERR_MISALIGNED;
  if ((st = check_state_aliases(in->H_k, in->H_v, N, state_in, state_out, conv_in, conv_out, out,
                                static_cast<size_t>(T_tot) * in->H_v * GDN_HEAD_DIM * sizeof(bf16))) != GDN_OK)
    return st;
  const size_t need = gdn_prefill_workspace_size(in->H_k, in->H_v, N, n_chunks);
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  if (states_in_workspace(in->H_k, in->H_v, N, state_in, state_out, conv_in, conv_out, workspace, need) ||
      overlap(out, static_cast<size_t>(T_tot) * in->H_v * GDN_HEAD_DIM * sizeof(bf16), workspace, need))
    return GDN_ERR_ALIAS;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  gdn::PrefillParams p = {};
  p.q = static_cast<const bf16*>(in->q);
  p.k = static_cast<const bf16*>(in->k);
  p.v = static_cast<const bf16*>(in->v);
  p.a = static_cast<const bf16*>(in->a);
  p.b = static_cast<const bf16*>(in->b);
  p.z = static_cast<const bf16*>(in->z);
  p.sq = in->stride_q; p.sk = in->stride_k; p.sv = in->stride_v; p.sz = in->stride_z;
  p.sa = in->stride_a; p.sb = in->stride_b;
  p.conv_w = static_cast<const bf16*>(in->conv_w);
  p.A_log = in->A_log;
  p.norm_w = static_cast<const bf16*>(in->norm_w);
  p.scale = in->scale;
  p.H_k = in->H_k;
  p.H_v = in->H_v;
  p.N = N;
  p.cu = cu;
  p.T_uniform = T_uniform;
  p.n_chunks = n_chunks;
  p.T_total = T_tot;
  p.ws_flag = reinterpret_cast<int*>(ws);
  p.chunk_base = cu ? reinterpret_cast<int*>(ws + gdn::kWsHeader) : nullptr;
  p.seq_order = cu ? reinterpret_cast<int*>(ws + gdn::kWsHeader) + (N + 1) : nullptr;
  p.ws_k = ws + gdn::kWsHeader + chunk_base_bytes(N);
  p.ws_head = p.ws_k + static_cast<size_t>(n_chunks) * in->H_k * gdn::kKBytes;
  p.ws_end = ws + need;  // the layout's own end (a caller may pass more)
  p.state_in = state_in;
  p.state_out = state_out;
  p.conv_in = static_cast<const bf16*>(conv_in);
  p.conv_out = static_cast<bf16*>(conv_out);
  p.out = static_cast<bf16*>(out);
  p.err = err;
  p.allow_fused = in->schedule == 0 ? 1 : in->schedule == 2 ? 2 : 0;
  cudaError_t e = gdn::launch_prefill(p, static_cast<cudaStream_t>(stream), in->events);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t gdn_prefill_workspace_size(int H_k, int H_v, int N, long long n_chunks) {
  if (H_k <= 0 || H_v <= 0 || N < 0 || n_chunks < 0) return 0;
  return gdn::kWsHeader + chunk_base_bytes(N) +
         static_cast<size_t>(n_chunks) * (static_cast<size_t>(H_k) * gdn::kKBytes +
                                          static_cast<size_t>(H_v) * gdn::kHeadBytes);
}

gdn_status gdn_prefill(const gdn_inputs* in, int B, int T, const float* state_in, float* state_out,
                       const void* conv_in, void* conv_out, void* out, void* workspace, size_t workspace_bytes,
                       int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_prefill");
  if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot > INT_MAX) return GDN_ERR_UNSUPPORTED;
  const long long n_chunks = static_cast<long long>(B) * ((T + GDN_CHUNK - 1) / GDN_CHUNK);
  return prefill_common(in, B, T_tot, n_chunks, nullptr, T, state_in, state_out, conv_in, conv_out, out, workspace,
                        workspace_bytes, err, stream);
}

gdn_status gdn_prefill_varlen(const gdn_inputs* in, int N, const int* cu_seqlens, const int* cu_seqlens_host,
                              const float* state_in, float* state_out, const void* conv_in, void* conv_out,
                              void* out, void* workspace, size_t workspace_bytes, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_prefill_varlen");
  if (N < 0) return GDN_ERR_INVALID_ARG;
  if (N == 0) return check_inputs(in, 0);
  if (!cu_seqlens || !cu_seqlens_host) return GDN_ERR_INVALID_ARG;
  if (cu_seqlens_host[0] != 0) return GDN_ERR_INVALID_ARG;
  long long n_chunks = 0;
  for (int n = 0; n < N; ++n) {
    const long long L = static_cast<long long>(cu_seqlens_host[n + 1]) - cu_seqlens_host[n];
    if (L < 0) return GDN_ERR_INVALID_ARG;
    n_chunks += (L + GDN_CHUNK - 1) / GDN_CHUNK;
  }
  if (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) return GDN_ERR_MISALIGNED;
  return prefill_common(in, N, cu_seqlens_host[N], n_chunks, cu_seqlens, 0, state_in, state_out, conv_in, conv_out,
                        out, workspace, workspace_bytes, err, stream);
}

// Device copies of gdn_prefill_host's host tensors, after the prefill workspace, each from a
// 1 KiB boundary: q, k, v, z, a, b packed [T_tot][channels], then state, conv_in, conv_out, out.
struct HostStage {
  size_t q, k, v, z, a, b, state, conv_in, conv_out, out, end;
};

static HostStage host_stage_layout(int H_k, int H_v, int B, int T) {
  const size_t T_tot = static_cast<size_t>(B) * T;
  const size_t qk = T_tot * H_k * GDN_HEAD_DIM * 2, vz = T_tot * H_v * GDN_HEAD_DIM * 2, ab = T_tot * H_v * 2;
  const size_t state = static_cast<size_t>(B) * H_v * GDN_HEAD_DIM * GDN_HEAD_DIM * 4;
  const size_t conv = static_cast<size_t>(B) * 3 * (2 * H_k + H_v) * GDN_HEAD_DIM * 2;
  const long long n_chunks = static_cast<long long>(B) * ((T + GDN_CHUNK - 1) / GDN_CHUNK);
  HostStage L;
  size_t o = round_up(gdn_prefill_workspace_size(H_k, H_v, B, n_chunks), 1024);
  L.q = o; o += round_up(qk, 1024);
  L.k = o; o += round_up(qk, 1024);
  L.v = o; o += round_up(vz, 1024);
  L.z = o; o += round_up(vz, 1024);
  L.a = o; o += round_up(ab, 1024);
  L.b = o; o += round_up(ab, 1024);
  L.state = o; o += round_up(state, 1024);
  L.conv_in = o; o += round_up(conv, 1024);
  L.conv_out = o; o += round_up(conv, 1024);
  L.out = o; o += round_up(vz, 1024);
  L.end = o;
  return L;
}

size_t gdn_prefill_host_workspace_size(int H_k, int H_v, int B, int T) {
  if (H_k <= 0 || H_v <= 0 || B < 0 || T < 0) return 0;
  return host_stage_layout(H_k, H_v, B, T).end;
}

gdn_status gdn_prefill_host(const gdn_inputs* in, int B, int T, const float* state_in, float* state_out,
                            const void* conv_in, void* conv_out, void* out, void* workspace, size_t workspace_bytes,
                            int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_prefill_host");
  if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot > INT_MAX) return GDN_ERR_UNSUPPORTED;
  gdn_status st = check_inputs(in, T_tot);
  if (st != GDN_OK) return st;
  if (B == 0) return GDN_OK;
  if (T_tot > 0 && !out) return GDN_ERR_INVALID_ARG;
  if (T_tot > 0 && (st = check_out_alias(in, T_tot, out)) != GDN_OK) return st;
  const HostStage S = host_stage_layout(in->H_k, in->H_v, B, T);
  if (!workspace || workspace_bytes < S.end) return GDN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDN_ERR_MISALIGNED;
  const size_t state_bytes = static_cast<size_t>(B) * in->H_v * GDN_HEAD_DIM * GDN_HEAD_DIM * sizeof(float);
  const size_t conv_bytes = static_cast<size_t>(B) * 3 * (2 * in->H_k + in->H_v) * GDN_HEAD_DIM * sizeof(bf16);
  const size_t out_bytes = static_cast<size_t>(T_tot) * in->H_v * GDN_HEAD_DIM * sizeof(bf16);
  if ((st = check_state_aliases(in->H_k, in->H_v, B, state_in, state_out, conv_in, conv_out, out, out_bytes)) !=
      GDN_OK)
    return st;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t qk_w = static_cast<size_t>(in->H_k) * GDN_HEAD_DIM, vz_w = static_cast<size_t>(in->H_v) * GDN_HEAD_DIM;
  // inputs in: one (strided) copy per tensor into its packed device copy
  struct Part { const void* src; long long stride; size_t width; size_t off; };
  const Part parts[6] = {{in->q, in->stride_q, qk_w, S.q}, {in->k, in->stride_k, qk_w, S.k},
                         {in->v, in->stride_v, vz_w, S.v}, {in->z, in->stride_z, vz_w, S.z},
                         {in->a, in->stride_a, static_cast<size_t>(in->H_v), S.a},
                         {in->b, in->stride_b, static_cast<size_t>(in->H_v), S.b}};
  if (T_tot > 0) {
    for (const Part& pt : parts) {
      if (cudaMemcpy2DAsync(ws + pt.off, pt.width * 2, pt.src, static_cast<size_t>(pt.stride) * 2, pt.width * 2,
                            static_cast<size_t>(T_tot), cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return GDN_ERR_CUDA;
    }
  }
  float* d_state = reinterpret_cast<float*>(ws + S.state);
  if (state_in && cudaMemcpyAsync(d_state, state_in, state_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (conv_in && cudaMemcpyAsync(ws + S.conv_in, conv_in, conv_bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess)
    return GDN_ERR_CUDA;
  // the prefill on the device copies (state updated in place)
  gdn_inputs d = *in;
  d.q = ws + S.q; d.k = ws + S.k; d.v = ws + S.v; d.z = ws + S.z; d.a = ws + S.a; d.b = ws + S.b;
  d.stride_q = d.stride_k = static_cast<long long>(qk_w);
  d.stride_v = d.stride_z = static_cast<long long>(vz_w);
  d.stride_a = d.stride_b = in->H_v;
  const long long n_chunks = static_cast<long long>(B) * ((T + GDN_CHUNK - 1) / GDN_CHUNK);
  st = prefill_common(&d, B, T_tot, n_chunks, nullptr, T, state_in ? d_state : nullptr,
                      state_out ? d_state : nullptr, conv_in ? ws + S.conv_in : nullptr,
                      conv_out ? ws + S.conv_out : nullptr, ws + S.out, workspace, workspace_bytes, err, stream);
  if (st != GDN_OK) return st;
  // outputs back
  if (T_tot > 0 && cudaMemcpyAsync(out, ws + S.out, out_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (state_out && cudaMemcpyAsync(state_out, d_state, state_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (conv_out && cudaMemcpyAsync(conv_out, ws + S.conv_out, conv_bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_OK;
}

gdn_status gdn_gemm_bf16(const void* A, long long lda, const void* B, long long ldb, void* C, long long ldc, int M,
                         int N, int K, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_gemm_bf16");
  if (M < 0 || N < 0 || K < 0) return GDN_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return GDN_OK;
  if (!A || !B || !C || K == 0) return GDN_ERR_INVALID_ARG;
  if (K % 64 != 0) return GDN_ERR_UNSUPPORTED;
  if (lda < K || ldb < K || ldc < N) return GDN_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C) || ((lda | ldb | ldc) & 7)) return GDN_ERR_MISALIGNED;
  const size_t a_bytes = (static_cast<size_t>(M - 1) * lda + K) * 2, b_bytes = (static_cast<size_t>(N - 1) * ldb + K) * 2;
  const size_t c_bytes = (static_cast<size_t>(M - 1) * ldc + N) * 2;
  if (overlap(C, c_bytes, A, a_bytes) || overlap(C, c_bytes, B, b_bytes)) return GDN_ERR_ALIAS;
  const cudaError_t e = gdn::launch_gemm_bf16(static_cast<const bf16*>(A), lda, static_cast<const bf16*>(B), ldb,
                                              static_cast<bf16*>(C), ldc, M, N, K, err,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

long long gdn_layer_n_in(int H_k, int H_v) {
  if (H_k <= 0 || H_v <= 0) return 0;
  return 2LL * H_k * GDN_HEAD_DIM + 2LL * H_v * GDN_HEAD_DIM + 2LL * H_v;
}

size_t gdn_layer_workspace_size(int H_k, int H_v, int B, int T) {
  if (H_k <= 0 || H_v <= 0 || B < 0 || T < 0) return 0;
  const long long T_tot = static_cast<long long>(B) * T;
  const long long n_chunks = static_cast<long long>(B) * ((T + GDN_CHUNK - 1) / GDN_CHUNK);
  const size_t proj = round_up(static_cast<size_t>(T_tot) * layer_ld_proj(H_k, H_v) * 2, 1024);
  const size_t mix = round_up(static_cast<size_t>(T_tot) * H_v * GDN_HEAD_DIM * 2, 1024);
  return proj + mix + gdn_prefill_workspace_size(H_k, H_v, B, n_chunks);
}

gdn_status gdn_layer_prefill(const gdn_layer* L, int B, int T, const void* x, long long ldx, const float* state_in,
                             float* state_out, const void* conv_in, void* conv_out, void* y, long long ldy,
                             void* workspace, size_t workspace_bytes, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_layer_prefill");
  if (!L || B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  if (L->H_k <= 0 || L->H_v <= 0 || L->hidden <= 0 || L->H_v % L->H_k != 0) return GDN_ERR_INVALID_ARG;
  if (L->hidden % 64 != 0) return GDN_ERR_UNSUPPORTED;
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot > INT_MAX) return GDN_ERR_UNSUPPORTED;
  if (T_tot == 0) return GDN_OK;
  if (!x || !y || !L->w_in || !L->w_out) return GDN_ERR_INVALID_ARG;
  gdn_status cs = check_layer_states(L->H_k, L->H_v, B, state_in, state_out, conv_in, conv_out);
  if (cs != GDN_OK) return cs;
  const size_t need = gdn_layer_workspace_size(L->H_k, L->H_v, B, T);
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  const long long n_in = gdn_layer_n_in(L->H_k, L->H_v), ld_p = layer_ld_proj(L->H_k, L->H_v);
  const long long d_v = static_cast<long long>(L->H_v) * GDN_HEAD_DIM;
  if (ldy < L->hidden) return GDN_ERR_INVALID_ARG;
  if (overlap(y, (static_cast<size_t>(T_tot - 1) * ldy + L->hidden) * 2, workspace, need)) return GDN_ERR_ALIAS;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  bf16* proj = reinterpret_cast<bf16*>(ws);
  bf16* mix = reinterpret_cast<bf16*>(ws + round_up(static_cast<size_t>(T_tot) * ld_p * 2, 1024));
  uint8_t* ws_mixer = reinterpret_cast<uint8_t*>(mix) + round_up(static_cast<size_t>(T_tot) * d_v * 2, 1024);
  const size_t ws_mixer_bytes = workspace_bytes - static_cast<size_t>(ws_mixer - ws);
  // everything the mixer call would reject is rejected here, before the first launch
  const gdn_inputs in = layer_mixer_inputs(L, proj, ld_p);
  if ((cs = check_inputs(&in, T_tot)) != GDN_OK) return cs;
  if (!aligned16(workspace)) return GDN_ERR_MISALIGNED;
  if (states_in_workspace(L->H_k, L->H_v, B, state_in, state_out, conv_in, conv_out, workspace, need))
    return GDN_ERR_ALIAS;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) {
    if (L->events) cudaEventRecord(static_cast<cudaEvent_t>(L->events[i]), st);
  };
  mark(0);
  gdn_status s = gdn_gemm_bf16(x, ldx, L->w_in, L->ld_w_in, proj, ld_p, static_cast<int>(T_tot),
                               static_cast<int>(n_in), L->hidden, err, stream);
  if (s != GDN_OK) return s;
  mark(1);
  s = gdn_prefill(&in, B, T, state_in, state_out, conv_in, conv_out, mix, ws_mixer, ws_mixer_bytes, err, stream);
  if (s != GDN_OK) return s;
  mark(2);
  s = gdn_gemm_bf16(mix, d_v, L->w_out, L->ld_w_out, y, ldy, static_cast<int>(T_tot), L->hidden,
                    static_cast<int>(d_v), err, stream);
  if (s != GDN_OK) return s;
  mark(3);
  return GDN_OK;
}

size_t gdn_layer_decode_workspace_size(int H_k, int H_v, int N, int T) {
  if (H_k <= 0 || H_v <= 0 || N < 0 || T < 1 || T > gdn::kMaxDecodeTokens) return 0;
  const size_t T_tot = static_cast<size_t>(N) * T;
  return round_up(T_tot * layer_ld_proj(H_k, H_v) * 2, 1024) +
         round_up(T_tot * static_cast<size_t>(H_v) * GDN_HEAD_DIM * 2, 1024);
}

gdn_status gdn_layer_decode(const gdn_layer* L, int N, int T, const void* x, long long ldx, float* state,
                            void* conv_state, const int* state_slot, int n_slots, void* y, long long ldy,
                            void* workspace, size_t workspace_bytes, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_layer_decode");
  if (!L || N < 0 || T < 1 || T > gdn::kMaxDecodeTokens) return GDN_ERR_INVALID_ARG;
  if (L->H_k <= 0 || L->H_v <= 0 || L->hidden <= 0 || L->H_v % L->H_k != 0) return GDN_ERR_INVALID_ARG;
  if (L->hidden % 64 != 0) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!x || !y || !L->w_in || !L->w_out || !state || !conv_state) return GDN_ERR_INVALID_ARG;
  if (state_slot && n_slots < 1) return GDN_ERR_INVALID_ARG;
  // decode updates both in place: they are the written buffers of the rule
  gdn_status cs = check_layer_states(L->H_k, L->H_v, state_slot ? n_slots : N, nullptr, state, nullptr, conv_state);
  if (cs != GDN_OK) return cs;
  const long long T_tot = static_cast<long long>(N) * T;
  const size_t need = gdn_layer_decode_workspace_size(L->H_k, L->H_v, N, T);
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  if (ldy < L->hidden) return GDN_ERR_INVALID_ARG;
  if (overlap(y, (static_cast<size_t>(T_tot - 1) * ldy + L->hidden) * 2, workspace, need)) return GDN_ERR_ALIAS;
  const long long n_in = gdn_layer_n_in(L->H_k, L->H_v), ld_p = layer_ld_proj(L->H_k, L->H_v);
  const long long d_v = static_cast<long long>(L->H_v) * GDN_HEAD_DIM;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  bf16* proj = reinterpret_cast<bf16*>(ws);
  bf16* mix = reinterpret_cast<bf16*>(ws + round_up(static_cast<size_t>(T_tot) * ld_p * 2, 1024));
  // everything the decode call would reject is rejected here, before the first launch
  const gdn_inputs in = layer_mixer_inputs(L, proj, ld_p);
  if ((cs = check_inputs(&in, T_tot)) != GDN_OK) return cs;
  if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(state_slot) & 3u)) return GDN_ERR_MISALIGNED;
  if (states_in_workspace(L->H_k, L->H_v, state_slot ? n_slots : N, state, nullptr, conv_state, nullptr, workspace,
                          need))
    return GDN_ERR_ALIAS;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) {
    if (L->events) cudaEventRecord(static_cast<cudaEvent_t>(L->events[i]), st);
  };
  mark(0);
  gdn_status s = gdn_gemm_bf16(x, ldx, L->w_in, L->ld_w_in, proj, ld_p, static_cast<int>(T_tot),
                               static_cast<int>(n_in), L->hidden, err, stream);
  if (s != GDN_OK) return s;
  mark(1);
  s = gdn_decode_multi(&in, N, T, state, conv_state, state_slot, state_slot ? n_slots : N, mix, err, stream);
  if (s != GDN_OK) return s;
  mark(2);
  s = gdn_gemm_bf16(mix, d_v, L->w_out, L->ld_w_out, y, ldy, static_cast<int>(T_tot), L->hidden,
                    static_cast<int>(d_v), err, stream);
  if (s != GDN_OK) return s;
  mark(3);
  return GDN_OK;
}

gdn_status gdn_attention_prefill(const void* q_hat, const void* k, const void* v, const void* g, long long ld_g,
                                 int B, int T, void* out, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_attention_prefill");
  if (B < 0 || T < 0) return GDN_ERR_INVALID_ARG;
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot > INT_MAX) return GDN_ERR_UNSUPPORTED;
  if (T_tot == 0) return GDN_OK;
  const long long hd = static_cast<long long>(GDN_ATTN_Q_HEADS) * GDN_ATTN_HEAD_DIM;
  if (!q_hat || !k || !v || !g || !out || ld_g < hd) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q_hat) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(out) || (ld_g & 7))
    return GDN_ERR_MISALIGNED;
  const size_t ob = static_cast<size_t>(T_tot) * hd * 2;
  const size_t kvb = static_cast<size_t>(T_tot) * GDN_ATTN_KV_HEADS * GDN_ATTN_HEAD_DIM * 2;
  if (overlap(out, ob, q_hat, ob) || overlap(out, ob, k, kvb) || overlap(out, ob, v, kvb) ||
      overlap(out, ob, g, (static_cast<size_t>(T_tot - 1) * ld_g + hd) * 2))
    return GDN_ERR_ALIAS;
  return gdn::launch_flash_attn(static_cast<const bf16*>(q_hat), static_cast<const bf16*>(k),
                                static_cast<const bf16*>(v), T, static_cast<const bf16*>(g), ld_g, B, T,
                                static_cast<bf16*>(out), err, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GDN_OK
             : GDN_ERR_CUDA;
}

size_t gdn_attn_layer_workspace_size(int B, int T) {
  if (B < 0 || T < 0) return 0;
  const size_t T_tot = static_cast<size_t>(B) * T;
  const size_t hd = static_cast<size_t>(GDN_ATTN_Q_HEADS) * GDN_ATTN_HEAD_DIM;
  return round_up(T_tot * GDN_ATTN_N_IN * 2, 1024) + 2 * round_up(T_tot * hd * 2, 1024);
}

gdn_status gdn_attn_layer_prefill(const gdn_attn_layer* L, int B, int T, const void* x, long long ldx,
                                  void* k_cache, void* v_cache, int cache_cap, void* y, long long ldy,
                                  void* workspace, size_t workspace_bytes, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_attn_layer_prefill");
  if (!L || B < 0 || T < 0 || L->hidden <= 0 || cache_cap < 0) return GDN_ERR_INVALID_ARG;
  const int cap = cache_cap == 0 ? T : cache_cap;
  if (cap < T) return GDN_ERR_INVALID_ARG;
  if (L->hidden % 64 != 0) return GDN_ERR_UNSUPPORTED;
  const long long T_tot = static_cast<long long>(B) * T;
  if (T_tot > INT_MAX) return GDN_ERR_UNSUPPORTED;
  if (T_tot == 0) return GDN_OK;
  if (!x || !y || !k_cache || !v_cache || !L->w_in || !L->w_out || !L->q_norm_w || !L->k_norm_w)
    return GDN_ERR_INVALID_ARG;
  if (ldy < L->hidden) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_attn_layer_workspace_size(B, T);
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(L->q_norm_w) || !aligned16(L->k_norm_w) ||
      !aligned16(workspace))
    return GDN_ERR_MISALIGNED;
  const size_t hd = static_cast<size_t>(GDN_ATTN_Q_HEADS) * GDN_ATTN_HEAD_DIM;
  const size_t kv_bytes = static_cast<size_t>(B) * cap * GDN_ATTN_KV_HEADS * GDN_ATTN_HEAD_DIM * 2;
  const size_t y_bytes = (static_cast<size_t>(T_tot - 1) * ldy + L->hidden) * 2;
  if (overlap(y, y_bytes, workspace, need) || overlap(k_cache, kv_bytes, workspace, need) ||
      overlap(v_cache, kv_bytes, workspace, need) || overlap(k_cache, kv_bytes, v_cache, kv_bytes) ||
      overlap(y, y_bytes, k_cache, kv_bytes) || overlap(y, y_bytes, v_cache, kv_bytes))
    return GDN_ERR_ALIAS;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  bf16* proj = reinterpret_cast<bf16*>(ws);
  bf16* q_hat = reinterpret_cast<bf16*>(ws + round_up(static_cast<size_t>(T_tot) * GDN_ATTN_N_IN * 2, 1024));
  bf16* att = reinterpret_cast<bf16*>(reinterpret_cast<uint8_t*>(q_hat) + round_up(static_cast<size_t>(T_tot) * hd * 2, 1024));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) {
    if (L->events) cudaEventRecord(static_cast<cudaEvent_t>(L->events[i]), st);
  };
  mark(0);
  gdn_status s = gdn_gemm_bf16(x, ldx, L->w_in, L->ld_w_in, proj, GDN_ATTN_N_IN, static_cast<int>(T_tot),
                               GDN_ATTN_N_IN, L->hidden, err, stream);
  if (s != GDN_OK) return s;
  mark(1);
  if (gdn::launch_attn_qk(proj, GDN_ATTN_N_IN, static_cast<const bf16*>(L->q_norm_w),
                          static_cast<const bf16*>(L->k_norm_w), B, T, nullptr, cap, q_hat,
                          static_cast<bf16*>(k_cache), static_cast<bf16*>(v_cache), err, st) != cudaSuccess ||
      gdn::launch_flash_attn(q_hat, static_cast<const bf16*>(k_cache), static_cast<const bf16*>(v_cache), cap,
                             proj + hd, GDN_ATTN_N_IN, B, T, att, err, st) != cudaSuccess)
    return GDN_ERR_CUDA;
  mark(2);
  s = gdn_gemm_bf16(att, static_cast<long long>(hd), L->w_out, L->ld_w_out, y, ldy, static_cast<int>(T_tot),
                    L->hidden, static_cast<int>(hd), err, stream);
  if (s != GDN_OK) return s;
  mark(3);
  return GDN_OK;
}

size_t gdn_attn_decode_workspace_size(int N, int cache_cap) {
  if (N < 0 || cache_cap < 0) return 0;
  const size_t hd = static_cast<size_t>(GDN_ATTN_Q_HEADS) * GDN_ATTN_HEAD_DIM;
  return round_up(static_cast<size_t>(N) * GDN_ATTN_N_IN * 2, 1024) + 2 * round_up(static_cast<size_t>(N) * hd * 2, 1024) +
         round_up(gdn::attn_decode_part_bytes(N, cache_cap), 1024);
}

gdn_status gdn_attn_layer_decode_step(const gdn_attn_layer* L, int N, const void* x, long long ldx, void* k_cache,
                                      void* v_cache, int cache_cap, int* cache_len, void* y, long long ldy,
                                      void* workspace, size_t workspace_bytes, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_attn_layer_decode_step");
  if (!L || N < 0 || cache_cap <= 0 || L->hidden <= 0) return GDN_ERR_INVALID_ARG;
  if (L->hidden % 64 != 0) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!x || !y || !k_cache || !v_cache || !cache_len || !L->w_in || !L->w_out || !L->q_norm_w || !L->k_norm_w)
    return GDN_ERR_INVALID_ARG;
  if (ldy < L->hidden) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_attn_decode_workspace_size(N, cache_cap);
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(L->q_norm_w) || !aligned16(L->k_norm_w) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(cache_len) & 3u))
    return GDN_ERR_MISALIGNED;
  const size_t hd = static_cast<size_t>(GDN_ATTN_Q_HEADS) * GDN_ATTN_HEAD_DIM;
  const size_t kv_bytes = static_cast<size_t>(N) * cache_cap * GDN_ATTN_KV_HEADS * GDN_ATTN_HEAD_DIM * 2;
  const size_t y_bytes = (static_cast<size_t>(N - 1) * ldy + L->hidden) * 2;
  if (overlap(y, y_bytes, workspace, need) || overlap(k_cache, kv_bytes, workspace, need) ||
      overlap(v_cache, kv_bytes, workspace, need) || overlap(k_cache, kv_bytes, v_cache, kv_bytes) ||
      overlap(y, y_bytes, k_cache, kv_bytes) || overlap(y, y_bytes, v_cache, kv_bytes))
    return GDN_ERR_ALIAS;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  bf16* proj = reinterpret_cast<bf16*>(ws);
  bf16* q_hat = reinterpret_cast<bf16*>(ws + round_up(static_cast<size_t>(N) * GDN_ATTN_N_IN * 2, 1024));
  bf16* att = reinterpret_cast<bf16*>(reinterpret_cast<uint8_t*>(q_hat) + round_up(static_cast<size_t>(N) * hd * 2, 1024));
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(att) + round_up(static_cast<size_t>(N) * hd * 2, 1024));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) {
    if (L->events) cudaEventRecord(static_cast<cudaEvent_t>(L->events[i]), st);
  };
  mark(0);
  gdn_status s = gdn_gemm_bf16(x, ldx, L->w_in, L->ld_w_in, proj, GDN_ATTN_N_IN, N, GDN_ATTN_N_IN, L->hidden, err,
                               stream);
  if (s != GDN_OK) return s;
  mark(1);
  if (gdn::launch_attn_qk(proj, GDN_ATTN_N_IN, static_cast<const bf16*>(L->q_norm_w),
                          static_cast<const bf16*>(L->k_norm_w), N, 1, cache_len, cache_cap, q_hat,
                          static_cast<bf16*>(k_cache), static_cast<bf16*>(v_cache), err, st) != cudaSuccess ||
      gdn::launch_attn_decode(q_hat, static_cast<const bf16*>(k_cache), static_cast<const bf16*>(v_cache),
                              cache_cap, cache_len, proj + hd, GDN_ATTN_N_IN, N, part, att, st) != cudaSuccess)
    return GDN_ERR_CUDA;
  mark(2);
  s = gdn_gemm_bf16(att, static_cast<long long>(hd), L->w_out, L->ld_w_out, y, ldy, N, L->hidden,
                    static_cast<int>(hd), err, stream);
  if (s != GDN_OK) return s;
  mark(3);
  return GDN_OK;
}

gdn_status gdn_decode_multi(const gdn_inputs* in, int N, int T, float* state, void* conv_state,
                            const int* state_slot, int n_slots, void* out, int* err, void* stream) {
  const NvtxRange nvtx_range("gdn_decode_multi");
  if (N < 0 || T < 1 || T > gdn::kMaxDecodeTokens || n_slots < 0) return GDN_ERR_INVALID_ARG;
  const long long T_tot = static_cast<long long>(N) * T;
  gdn_status st = check_inputs(in, T_tot);
  if (st != GDN_OK || N == 0) return st;
  if (!state || !conv_state || !out) return GDN_ERR_INVALID_ARG;
  if (!state_slot && n_slots < N) return GDN_ERR_INVALID_ARG;  // slot n for sequence n
  if (!aligned16(state) || !aligned16(conv_state) || !aligned16(out)) return GDN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(state_slot) & 3u) return GDN_ERR_MISALIGNED;
  if ((st = check_out_alias(in, T_tot, out)) != GDN_OK) return st;
  const long long C_conv = static_cast<long long>(2 * in->H_k + in->H_v) * GDN_HEAD_DIM;
  const size_t state_bytes = static_cast<size_t>(n_slots) * in->H_v * GDN_HEAD_DIM * GDN_HEAD_DIM * sizeof(float);
  const size_t conv_bytes = static_cast<size_t>(n_slots) * 3 * C_conv * sizeof(bf16);
  const size_t out_bytes = static_cast<size_t>(T_tot) * in->H_v * GDN_HEAD_DIM * sizeof(bf16);
  if (overlap(state, state_bytes, conv_state, conv_bytes) || overlap(state, state_bytes, out, out_bytes) ||
      overlap(conv_state, conv_bytes, out, out_bytes))
    return GDN_ERR_ALIAS;
  gdn::DecodeParams p = {};
  p.q = static_cast<const bf16*>(in->q);
  p.k = static_cast<const bf16*>(in->k);
  p.v = static_cast<const bf16*>(in->v);
  p.a = static_cast<const bf16*>(in->a);
  p.b = static_cast<const bf16*>(in->b);
  p.z = static_cast<const bf16*>(in->z);
  p.sq = in->stride_q; p.sk = in->stride_k; p.sv = in->stride_v; p.sz = in->stride_z;
  p.sa = in->stride_a; p.sb = in->stride_b;
  p.conv_w = static_cast<const bf16*>(in->conv_w);
  p.A_log = in->A_log;
  p.norm_w = static_cast<const bf16*>(in->norm_w);
  p.scale = in->scale;
  p.H_k = in->H_k;
  p.H_v = in->H_v;
  p.N = N;
  p.T = T;
  p.state_slot = state_slot;
  p.n_slots = n_slots;
  p.state = state;
  p.conv_state = static_cast<bf16*>(conv_state);
  p.out = static_cast<bf16*>(out);
  p.err = err;
  return gdn::launch_decode(p, static_cast<cudaStream_t>(stream), in->events) == cudaSuccess ? GDN_OK
                                                                                         : GDN_ERR_CUDA;
}

gdn_status gdn_decode_step(const gdn_inputs* in, int N, float* state, void* conv_state, void* out, int* err,
                           void* stream) {
  const NvtxRange nvtx_range("gdn_decode_step");
  return gdn_decode_multi(in, N, 1, state, conv_state, nullptr, N, out, err, stream);
}

gdn_status gdn_err_status(int err_word) {
  if (err_word == 0) return GDN_OK;
  if (err_word & gdn::kDevErrTimeout) return GDN_ERR_DEVICE_TIMEOUT;
  return GDN_ERR_INVALID_ARG;
}

const char* gdn_status_string(gdn_status status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: null pointer, bad count or bad shape";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: request outside what this library implements";
    case GDN_ERR_MISALIGNED: return "GDN_ERR_MISALIGNED: pointer or stride not suitably aligned";
    case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS: buffers that must be distinct overlap";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA launch failed";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT: a bounded device-side wait gave up (err bit 1)";
    case GDN_ERR_WORKSPACE: return "GDN_ERR_WORKSPACE: workspace missing or too small";
  }
  return "unknown gdn_status";
}

}  // extern "C"
