// Launch parameters of the mixer kernels (internal to libgdn.so).
#pragma once

#include "gdn_ptx.cuh"

namespace gdn {

using bf16 = __nv_bfloat16;

// Per-chunk workspace written by the prep kernel and read by the scan kernel.
// Every tensor-core operand is stored as a bf16 pair (hi = bf16(x), lo =
// bf16(x - hi)) so that products keep ~16 significant bits:
//   per (chunk, key head):   [Q;K] operand image, 128 rows x 128, SW128 K-major: hi, then lo
//   per (chunk, value head): [P T~; T~] image (128 x 64, SW128 K-major): hi, then lo;
//                            v_hat fp32 (64 tokens x 128, four 32-wide column blocks);
//                            gates fp32 (gamma[64], decay-to-end[64], gamma_C)
constexpr int kQKImg = 32768;                                // one bf16 image
constexpr int kQKBytes = 2 * kQKImg;                         // hi + lo
constexpr int kPTImg = 16384;
constexpr int kPTBytes = 2 * kPTImg;
constexpr int kVBytes = 64 * 128 * 4;                        // fp32
constexpr int kGateBytes = 1024;
constexpr int kHeadBytes = kPTBytes + kVBytes + kGateBytes;  // 66560
constexpr int kWsHeader = 1024;                              // error/consistency word

struct DecodeParams {
  const bf16 *q, *k, *v, *a, *b, *z;
  long long sq, sk, sv, sz, sa, sb;  // token strides (elements)
  const bf16* conv_w;
  const float* A_log;
  const bf16* norm_w;
  float scale;
  int H_k, H_v, N;
  float* state;     // [N][H_v][128][128], updated in place
  bf16* conv_state; // [N][3][C_conv], updated in place
  bf16* out;        // [N][H_v][128]
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
  uint8_t* ws_qk;         // [n_chunks][H_k][kQKBytes]
  uint8_t* ws_head;       // [n_chunks][H_v][kHeadBytes]
  const float* state_in;  // [N][H_v][128][128] or null (zeros)
  float* state_out;       // [N][H_v][128][128] or null
  const bf16* conv_in;    // [N][3][C_conv] or null (zeros)
  bf16* conv_out;         // [N][3][C_conv] or null
  bf16* out;              // [T_tot][H_v][128]
  int* err;
};

// events: null, or cudaEvent_t handles recorded around the kernels (see gdn_inputs.events)
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream, void* const* events);
// dv_slice: 64 or 32 value rows of the state per scan CTA (a cluster of 128/dv_slice CTAs per head)
cudaError_t launch_prefill(const PrefillParams& p, int dv_slice, cudaStream_t stream, void* const* events);

}  // namespace gdn
