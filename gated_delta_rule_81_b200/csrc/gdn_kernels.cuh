// Launch parameters of the mixer kernels (internal to libgdn.so).
#pragma once

#include "gdn_ptx.cuh"

namespace gdn {

using bf16 = __nv_bfloat16;

// Per-chunk workspace written by the prep kernel and read by the scan kernel.
// Every tensor-core operand is stored as a bf16 pair (hi = bf16(x), lo =
// bf16(x - hi)) so that products keep ~16 significant bits.  Operand images use
// the 128-byte swizzled layout (rows of 64 bf16 = 128 B, 8-row groups of 1 KiB).
//   per (chunk, key head), kKBytes:
//     K hi | K lo: 64 tokens x 128 channels each, as two 8 KiB blocks of 64 channels
//     (row = token), read by the scan as an MN-major operand (N = channels).
//   per (chunk, value head), kHeadBytes:
//     -W^T lo | -W^T hi | (gamma Q)^T hi | (gamma Q)^T lo: four 16 KiB images of 128 rows
//       (d_k) x 64 tokens, W = T diag(beta gamma) K (negated) and gamma Q = diag(gamma) Q;
//       read by the scan as MN-major operands of N = 128 (-W^T lo | hi, -W^T hi | (gamma Q)^T hi,
//       (gamma Q)^T hi | lo)
//     P hi | P lo: P_ij = e^{G_i - G_j} q_i.k_j for j <= i, row = i, 64 j per row
//     B_U lo | B_U hi: B_U = T diag(beta), row = i, 64 j per row (K-major); side by side
//       one operand of N = 128
//     v_hat hi | v_hat lo: v_hat = SiLU(conv(v)) of the head, 64 token rows x 128 channels as
//       two 8 KiB blocks of 64 channels each (read by the scan as an MN-major operand, M = d_v)
//     gates fp32: gamma_i [64], e^{G_C - G_i} [64], gamma_C
constexpr int kImg64 = 16384;                                // 64 rows x 128 channels (or 128 x 64), bf16
constexpr int kKBytes = 2 * kImg64;                          // K hi, K lo
constexpr int kHeadOffW = 0;                                 // -W^T lo, -W^T hi
constexpr int kWBytes = 2 * kImg64;
constexpr int kHeadOffGQ = kHeadOffW + kWBytes;              // (gamma Q)^T hi, lo
constexpr int kPImg = 8192;                                  // one 64 x 64 bf16 image
constexpr int kHeadOffP = kHeadOffGQ + 2 * kImg64;           // P hi, lo
constexpr int kHeadOffBU = kHeadOffP + 2 * kPImg;            // B_U lo, hi
constexpr int kHeadOffV = kHeadOffBU + 2 * kPImg;            // v_hat hi, lo
constexpr int kHeadOffGate = kHeadOffV + 2 * kImg64;
constexpr int kGateBytes = 1024;
constexpr int kReadyFlagWord = 255;  // word of the gate area a fused prefill launch uses as a ready flag
constexpr int kHeadBytes = kHeadOffGate + kGateBytes;        // 132096
constexpr int kWsHeader = 1024;                              // error/consistency word

constexpr int kMaxDecodeTokens = 8;   // new tokens per sequence in one decode call
constexpr int kDevErrBadSlot = 8;      // a state_slot entry outside [0, n_slots)

struct DecodeParams {
  const bf16 *q, *k, *v, *a, *b, *z;  // token n * T + t is new token t of sequence n
  long long sq, sk, sv, sz, sa, sb;   // token strides (elements)
  const bf16* conv_w;
  const float* A_log;
  const bf16* norm_w;
  float scale;
  int H_k, H_v, N;
  int T;                  // new tokens per sequence, 1 .. kMaxDecodeTokens
  const int* state_slot;  // [N] slot of each sequence in the state pools, or null (slot n)
  int n_slots;            // slots in the pools
  float* state;           // [n_slots][H_v][128][128], updated in place
  bf16* conv_state;       // [n_slots][3][C_conv], updated in place
  bf16* out;              // [N * T][H_v][128]
  int* err;
};

struct PrefillParams {
  const bf16 *q, *k, *v, *a, *b, *z;
  long long sq, sk, sv, sz, sa, sb;
  const bf16* conv_w;
  const float* A_log;
  const bf16* norm_w;
  float scale;
  int H_k, H_v;
  int N;                  // sequences
  const int* cu;          // device cu_seqlens [N+1], or null for uniform length T_uniform
  int T_uniform;
  long long n_chunks;     // total chunks (host count)
  long long T_total;      // total tokens (host count)
  int* chunk_base;        // [N+1] in the workspace (varlen), or null (uniform)
  int* seq_order;         // [N] scan order, longest first (varlen), or null
  int* ws_flag;           // workspace header word: nonzero = inconsistent cu_seqlens
  uint8_t* ws_k;          // [n_chunks][H_k][kKBytes]
  uint8_t* ws_head;       // [n_chunks][H_v][kHeadBytes]
  const uint8_t* ws_end;  // one past the caller's workspace (checked by the debug build)
  const float* state_in;  // [N][H_v][128][128] or null (zeros)
  float* state_out;       // [N][H_v][128][128] or null
  const bf16* conv_in;    // [N][3][C_conv] or null (zeros)
  bf16* conv_out;         // [N][3][C_conv] or null
  bf16* out;              // [T_tot][H_v][128]
  int* err;
  int allow_fused;        // 0 = two launches, 1 = automatic, 2 = one fused launch whenever possible
  int fused_scan_ctas;    // set by launch_prefill: > 0 = one fused launch, the scan on its last CTAs,
                          // prep items published by ready flags; 0 = prep kernel, then scan kernel
};

constexpr int kDevErrBounds = 64;  // (debug build) an access outside the workspace was skipped

// Debug build (GDN_DEBUG, libgdn_debug.so): every workspace access of the prefill kernels is
// checked against [ws_k, ws_end); one outside sets kDevErrBounds and is skipped (never a trap).
// In the product build the check is the constant true and compiles away.
#ifdef GDN_DEBUG
__device__ __forceinline__ bool ws_ok(const PrefillParams& p, const void* ptr, long long bytes) {
  const uint8_t* a = static_cast<const uint8_t*>(ptr);
  const bool ok = a >= p.ws_k && bytes >= 0 && a + bytes <= p.ws_end;
  if (!ok && p.err) atomicOr(p.err, kDevErrBounds);
  return ok;
}
#else
__device__ __forceinline__ constexpr bool ws_ok(const PrefillParams&, const void*, long long) { return true; }
#endif

// events: null, or cudaEvent_t handles recorded around the kernels (see gdn_inputs.events)
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream, void* const* events);
cudaError_t launch_prefill(const PrefillParams& p, cudaStream_t stream, void* const* events);
// C[M][N] = A[M][K] B[N][K]^T in bf16 with fp32 accumulation (row-major, leading dimensions
// in elements; K a multiple of 64; pointers and leading dimensions 16-byte aligned).  Up to
// kGemvMaxM rows of A go through a weight-streaming kernel, more through tcgen05 tiles.
constexpr int kGemvMaxM = 4;
cudaError_t launch_gemm_bf16(const bf16* A, long long lda, const bf16* B, long long ldb, bf16* C, long long ldc,
                             int M, int N, int K, int* err, cudaStream_t stream);
// The global-attention layer between its projections.
// launch_attn_qk: proj [N T][ld_p] holds q (24 x 256) | g (24 x 256) | k (4 x 256) | v (4 x 256) of
// T tokens for each of N sequences; writes q_hat [N T][24][256] and k_hat, v into the caches
// [N][cap][4][256] at rows (pos_base ? pos_base[n] : 0) + t (error bit 16 past the capacity).
cudaError_t launch_attn_qk(const bf16* proj, long long ld_p, const bf16* q_norm_w, const bf16* k_norm_w, int N,
                           int T, const int* pos_base, int cap, bf16* q_hat, bf16* k_cache, bf16* v_cache, int* err,
                           cudaStream_t stream);
// launch_flash_attn: out [B T][24 x 256] = causal softmax(q_hat k^T / 16) v * sigmoid(g), GQA 24 / 4, with
// k, v the caches [B][kv_cap][4][256] (their first T rows); g: head h of token t at g + t * ld_g + h * 256.
cudaError_t launch_flash_attn(const bf16* q_hat, const bf16* k, const bf16* v, int kv_cap, const bf16* g,
                              long long ld_g, int B, int T, bf16* out, int* err, cudaStream_t stream);
// Decode: one new token per sequence already in the caches at row cache_len[n]; out [N][24 x 256];
// part: scratch of attn_decode_part_bytes(N, cap); cache_len advanced by one on the stream.
size_t attn_decode_part_bytes(int N, int cap);
cudaError_t launch_attn_decode(const bf16* q_hat, const bf16* k_cache, const bf16* v_cache, int cap, int* cache_len,
                               const bf16* g, long long ld_g, int N, float* part, bf16* out, cudaStream_t stream);

}  // namespace gdn
