/*
 * gdn.h -- C ABI of the B200 (sm_100a) gated-delta-rule token mixer.
 *
 * The mixer is the recurrent token mixer of the hybrid decoder described on
 * the Agnes-3.0-Flash pages: model card, "Architecture" table, row
 * "Delta-rule layers" (16 key heads / 48 value heads, head dim 128, a causal
 * conv of kernel 4 in front, a gated RMS-norm after, recurrent state in fp32);
 * "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model",
 * section "Feed-Forward and Positional Encoding", paragraph on the Gated Delta
 * Rule (each step erases the key's old association and then writes the new
 * value, and a forget gate decays the memory).  Per value head h (key head h / (H_v / H_k)) and token t:
 *
 *   x_t      = [q | k | v] raw channels; y = SiLU(causal depthwise conv_4(x))
 *   q_t, k_t = per-head L2-normalised y (x / sqrt(sum x^2 + 1e-6)), q_t *= scale
 *   g_t      = -exp(A_log[h]) * softplus(a_t),  alpha_t = exp(g_t),  beta_t = sigmoid(b_t)
 *   S_t      = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T   (S: d_v x d_k, fp32)
 *   o_t      = S_t q_t
 *   out_t    = o_t / sqrt(mean(o_t^2) + 1e-6) * norm_w * SiLU(z_t)           (bf16, RNE)
 *
 * Conventions common to every call:
 *   - All tensor pointers are DEVICE pointers unless named *_host.  The caller
 *     owns every buffer; the library keeps no state between calls and
 *     allocates no memory (prefill scratch is the caller's `workspace`).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise.  A returned GDN_OK means the work was
 *     validated and launched.
 *   - Head dim is fixed at 128 (GDN_HEAD_DIM), H_v % H_k == 0 and
 *     1 <= H_v / H_k <= 8.  Every tensor base pointer and every token stride
 *     (in bytes) must be a multiple of 16.
 *   - Layouts: q, k [T_tot][stride_q|k] with the H_k*128 head channels first;
 *     v, z [T_tot][stride_v|z] with H_v*128 channels; a, b [T_tot][stride_a|b]
 *     with H_v gate logits; out [T_tot][H_v][128] contiguous.  All bf16.
 *     conv_w bf16 [C_conv][4] with C_conv = (2 H_k + H_v) * 128 channels
 *     ordered q | k | v and tap 3 applied to the current token; A_log fp32
 *     [H_v]; norm_w bf16 [128] shared by all heads.
 *   - Recurrent state: fp32 [N][H_v][128 (d_v)][128 (d_k)], row-major.
 *     Conv state: bf16 [N][3][C_conv], the 3 most recent raw tokens, oldest first.
 *   - `err` (nullable) is a device int the kernels OR error bits into
 *     (1 = a bounded wait timed out, 2 = reserved,
 *     4 = cu_seqlens on the device disagreed with cu_seqlens_host, 8 = a decode
 *     state_slot outside the pool, 16 = an attention KV cache with no row left, 32 = an
 *     attention decode cache_len outside [0, cache_cap], 64 = (libgdn_debug.so only) a
 *     prefill kernel found a workspace access outside the workspace and skipped it).
 *     It is never cleared by the library.  Read it after synchronising; gdn_err_status
 *     maps it to a gdn_status.
 *   - libgdn_debug.so exports the same calls, built with every workspace access of the
 *     prefill kernels checked against the workspace's bounds (a failed check sets bit 64
 *     and skips the access; nothing traps).  Same results as libgdn.so on valid calls.
 *   - With GDN_NVTX set in the environment (to anything but "0", read on the first
 *     call), every launching entry point pushes an NVTX range named after itself for
 *     its duration on the host (NVTX3, header-only: nothing is loaded unless a
 *     profiler injects its library).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_HEAD_DIM 128
#define GDN_CHUNK 64
#define GDN_CONV_TAPS 4

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,   /* null required pointer, bad count, bad shape */
  GDN_ERR_UNSUPPORTED = 2,   /* valid request this library does not implement */
  GDN_ERR_MISALIGNED = 3,    /* a pointer or stride is not 16-byte aligned */
  GDN_ERR_ALIAS = 4,         /* buffers that must be distinct overlap */
  GDN_ERR_CUDA = 5,          /* a CUDA launch failed */
  GDN_ERR_DEVICE_TIMEOUT = 6,/* a bounded device-side wait gave up (bit 1 of *err): every call is
                                asynchronous, so no call returns it; gdn_err_status maps the word */
  GDN_ERR_WORKSPACE = 7      /* workspace null or smaller than required */
} gdn_status;

/* Per-token inputs and per-layer parameters shared by all entry points. */
typedef struct {
  const void* q;          /* bf16 [T_tot] x stride_q, first H_k*128 channels used (pre-conv) */
  const void* k;          /* bf16 [T_tot] x stride_k (pre-conv) */
  const void* v;          /* bf16 [T_tot] x stride_v, first H_v*128 channels used (pre-conv) */
  const void* a;          /* bf16 [T_tot] x stride_a, H_v decay logits */
  const void* b;          /* bf16 [T_tot] x stride_b, H_v beta logits */
  const void* z;          /* bf16 [T_tot] x stride_z, H_v*128 output-gate channels */
  long long stride_q, stride_k, stride_v, stride_z, stride_a, stride_b; /* token strides, elements */
  const void* conv_w;     /* bf16 [C_conv][4] */
  const float* A_log;     /* fp32 [H_v] */
  const void* norm_w;     /* bf16 [128] */
  int H_k, H_v;
  float scale;            /* multiplies the normalised q; 1.0 = o_t = S_t q_t as written above */
  void* const* events;    /* optional timing hook (benchmarking and profiling; NULL in normal use -- an
                             addition to the plain tensor arguments of the mixer calls, kept in the
                             struct so that timing a call does not need a second entry point):
                             NULL, or caller-created cudaEvent_t handles that
                             the library records on `stream` around its kernels.  Prefill: 3 events,
                             [0] before the prep kernel, [1] between prep and scan, [2] after the
                             scan; when both phases run as one fused launch (see `schedule`), [1] is
                             recorded right after [0] and [2] after the launch.  Decode: 2 events,
                             before and after the decode kernel. */
  int schedule;           /* prefill launch plan.  1 = the chunk-parallel prep kernel, then the
                             sequential scan kernel.  2 = one launch that overlaps them chunk by
                             chunk (the scan on the launch's last CTAs, the prep on the others
                             publishing each chunk to the scan) whenever the scan's (sequence,
                             value head) units fit in half the SMs, else as 1.  0 = automatic: as 2 when the prep
                             also has at least 8 (chunk, key head) items per remaining SM, else
                             as 1.  "The SMs" are those the calling context may use (see
                             gdn_prefill_fused_plan).  Results are bitwise identical under every
                             plan. */
} gdn_inputs;

/*
 * The launch plan of a prefill: the number of scan CTAs of one overlapped launch, or 0 when
 * the prep and the scan run as two launches, for N sequences of n_chunks chunks in all, under
 * gdn_inputs.schedule `schedule`, on n_sm SMs.  The overlapped launch needs its scan CTAs
 * (N * H_v) to fit in half the SMs, so that the prep, which the scan waits for, always has SMs
 * of its own; the automatic plan (0) also wants at least 8 prep items (chunk, key head) per
 * remaining SM.  The prefill calls take n_sm from the calling context: the SMs of its SM
 * resource (a green context holds a partition of the device), scaled down by
 * CUDA_MPS_ACTIVE_THREAD_PERCENTAGE when that is set, else the device's count.  Pure host
 * function; 0 on bad arguments.
 */
int gdn_prefill_fused_plan(int H_k, int H_v, int N, long long n_chunks, int schedule, int n_sm);

/*
 * Bytes of device workspace gdn_prefill / gdn_prefill_varlen need for a batch
 * of N sequences that splits into n_chunks chunks of 64 tokens
 * (n_chunks = sum over sequences of ceil(L_n / 64)).  0 on bad arguments.
 */
size_t gdn_prefill_workspace_size(int H_k, int H_v, int N, long long n_chunks);

/*
 * Prefill of B sequences of T tokens each, packed as [B*T] tokens (sequence n
 * holds tokens n*T .. n*T+T-1).  Computes out for every token, and optionally
 * the final recurrent state and conv state of each sequence.
 * Departure from a launch that needs nothing but the tensors: the prefill takes a caller
 * `workspace`.  Its chunk-parallel phase (front end, triangular solve and the state-independent
 * products of every chunk, on all SMs at once) hands each chunk's operands to the sequential
 * phase through that scratch, which the library does not allocate itself (see
 * gdn_prefill_noalloc for callers that cannot provide one).  Both phases are described under
 * gdn_inputs.schedule.
 *   state_in   fp32 [B][H_v][128][128] or NULL (zero initial state)
 *   state_out  fp32 [B][H_v][128][128] or NULL; may equal state_in (in place)
 *   conv_in    bf16 [B][3][C_conv] or NULL (zero history)
 *   conv_out   bf16 [B][3][C_conv] or NULL; must not overlap conv_in
 *   out        bf16 [B*T][H_v][128]
 *   workspace  device scratch of gdn_prefill_workspace_size(H_k, H_v, B, B*ceil(T/64))
 *              bytes, 16-byte aligned; contents need no initialisation
 * B = 0 or T = 0 is a no-op apart from state_out = state_in and conv_out = conv_in history.
 */
gdn_status gdn_prefill(const gdn_inputs* in, int B, int T, const float* state_in, float* state_out,
                       const void* conv_in, void* conv_out, void* out, void* workspace,
                       size_t workspace_bytes, int* err, void* stream);

/*
 * gdn_prefill for tensors that live in host memory.  The per-token inputs q, k, v, a, b, z
 * of `in` (with its token strides), state_in, state_out, conv_in, conv_out and out are HOST
 * pointers, page-locked for the copies to run asynchronously; conv_w, A_log and norm_w stay
 * device pointers (the layer's weights live on the GPU).  On `stream`, in order: one copy
 * per input tensor into packed device copies held in `workspace` (after the prefill's own
 * scratch), gdn_prefill on them (the state updated in place on the device), one copy per
 * output back to the host.  Semantics, nullable arguments and errors as gdn_prefill; the
 * host buffers must stay valid and unmodified until the stream has passed the call.  Two
 * calls on two streams with two workspaces overlap one call's input copies with the other's
 * compute and output copies (the host link is full duplex).
 *   workspace  device memory of gdn_prefill_host_workspace_size(H_k, H_v, B, T) bytes,
 *              16-byte aligned, owned by the caller.
 */
size_t gdn_prefill_host_workspace_size(int H_k, int H_v, int B, int T);
gdn_status gdn_prefill_host(const gdn_inputs* in, int B, int T, const float* state_in, float* state_out,
                            const void* conv_in, void* conv_out, void* out, void* workspace,
                            size_t workspace_bytes, int* err, void* stream);

/*
 * Prefill of N variable-length sequences packed back to back.
 *   cu_seqlens       device int32 [N+1], cu[0] = 0, non-decreasing; sequence n is
 *                    tokens cu[n] .. cu[n+1]-1
 *   cu_seqlens_host  host copy of the same values (used to size the launch);
 *                    validated on the host.  The device copy is checked on the
 *                    device: cu[0] = 0, non-decreasing, and the same number of
 *                    chunks and total tokens as the host copy (otherwise nothing
 *                    is computed and *err gets bit 4)
 * Every sequence starts from its own state_in[n] / conv_in[n] (or zeros): state
 * and conv history never cross a cu_seqlens boundary.  Results for sequence n
 * are bitwise identical to a gdn_prefill of that sequence alone.  Other arguments as in gdn_prefill with leading dimension N; the
 * workspace size uses n_chunks = sum ceil((cu[n+1]-cu[n]) / 64).
 */
gdn_status gdn_prefill_varlen(const gdn_inputs* in, int N, const int* cu_seqlens,
                              const int* cu_seqlens_host, const float* state_in, float* state_out,
                              const void* conv_in, void* conv_out, void* out, void* workspace,
                              size_t workspace_bytes, int* err, void* stream);

/*
 * One decode step for N sequences, one new token each (token n of the inputs
 * belongs to sequence n, so T_tot = N).  Updates, in place,
 *   state       fp32 [N][H_v][128][128]
 *   conv_state  bf16 [N][3][C_conv]  (shifted by one token)
 * and writes out bf16 [N][H_v][128].  Inputs must not overlap state, conv_state or out.
 */
gdn_status gdn_decode_step(const gdn_inputs* in, int N, float* state, void* conv_state, void* out,
                           int* err, void* stream);

/*
 * The dense projections on either side of the mixer (hidden size 5120 -> q|k|v|z|a|b,
 * and 48*128 -> 5120; model card "Agnes-3.0-Flash Preview", "Architecture" table, rows
 * "Hidden size" and "Delta-rule layers"): C = A B^T on the tensor cores, bf16 in and out,
 * fp32 accumulation, one rounding to bf16 per output element.
 *   A  bf16 [M][lda], first K columns used        (activations, row-major)
 *   B  bf16 [N][ldb], first K columns used        (weights, one output channel per row)
 *   C  bf16 [M][ldc], first N columns written
 * K must be a multiple of 64 (GDN_ERR_UNSUPPORTED otherwise); every pointer and
 * leading dimension 16-byte aligned (GDN_ERR_MISALIGNED); C must not overlap A or
 * B (GDN_ERR_ALIAS).  M or N = 0 is a no-op.  Error bit 1 of *err: a wait inside
 * the kernel timed out.
 */
gdn_status gdn_gemm_bf16(const void* A, long long lda, const void* B, long long ldb, void* C, long long ldc, int M,
                         int N, int K, int* err, void* stream);

/*
 * One delta-rule layer around the mixer: y = out_proj(mixer(in_proj(x))) (model card
 * "Agnes-3.0-Flash Preview", "Architecture" table: hidden size 5120, delta-rule layers of
 * 16 key / 48 value heads of 128).  The pages give no layout for the projections; this
 * library's reading: the input projection's output channels are q (H_k*128) | k (H_k*128) |
 * v (H_v*128) | z (H_v*128) | a (H_v) | b (H_v), n_in of them in all; no biases.
 */
typedef struct {
  const void* w_in;       /* bf16 [n_in][ld_w_in], first `hidden` columns used */
  long long ld_w_in;
  const void* w_out;      /* bf16 [hidden][ld_w_out], first H_v*128 columns used */
  long long ld_w_out;
  const void* conv_w;     /* bf16 [C_conv][4] */
  const float* A_log;     /* fp32 [H_v] */
  const void* norm_w;     /* bf16 [128] */
  int H_k, H_v;
  int hidden;             /* model width; a multiple of 64 */
  float scale;            /* as gdn_inputs.scale */
  int schedule;           /* as gdn_inputs.schedule */
  void* const* events;    /* optional timing hook: NULL, or 4 caller-created cudaEvent_t recorded on
                             `stream` before the input projection, after it, after the mixer, and
                             after the output projection */
} gdn_layer;

/* Channels of the input projection's output: 2 H_k 128 + 2 H_v 128 + 2 H_v. */
long long gdn_layer_n_in(int H_k, int H_v);

/* Bytes of workspace gdn_layer_prefill needs for B sequences of T tokens: the
   projection output (bf16 [B T][n_in, padded to 8]), the mixer output (bf16 [B T][H_v 128])
   and the mixer's own workspace.  0 on bad arguments. */
size_t gdn_layer_workspace_size(int H_k, int H_v, int B, int T);

/*
 * Prefill of one delta-rule layer for B sequences of T tokens (packed [B*T]):
 *   x  bf16 [B*T][ldx], first `hidden` columns used;  y  bf16 [B*T][ldy], first `hidden` written.
 * state_in / state_out / conv_in / conv_out as in gdn_prefill.  Three launches
 * groups on `stream`: gdn_gemm_bf16 (in_proj), gdn_prefill on the projection's
 * columns (no copy: strided inputs), gdn_gemm_bf16 (out_proj).  Errors as those calls;
 * y must not overlap x or the workspace.
 */
gdn_status gdn_layer_prefill(const gdn_layer* L, int B, int T, const void* x, long long ldx, const float* state_in,
                             float* state_out, const void* conv_in, void* conv_out, void* y, long long ldy,
                             void* workspace, size_t workspace_bytes, int* err, void* stream);

/* Workspace bytes of gdn_layer_decode for N sequences of T new tokens (0 on bad arguments). */
size_t gdn_layer_decode_workspace_size(int H_k, int H_v, int N, int T);

/*
 * Decode of one delta-rule layer: T = 1 .. GDN_MAX_DECODE_TOKENS new tokens for each of N
 * sequences (x bf16 [N*T][ldx], token n*T + t = new token t of sequence n) -> y bf16
 * [N*T][ldy].  Three launch groups on `stream`: gdn_gemm_bf16 (in_proj), gdn_decode_multi on
 * the projection's columns (strided, no copy) with the states in place, gdn_gemm_bf16
 * (out_proj).  state, conv_state, state_slot and n_slots as in gdn_decode_multi (state_slot
 * NULL: sequence n uses slot n and n_slots is ignored).  A state left by gdn_layer_prefill
 * (state_out, conv_out) continues here unchanged: the handoff from prefill to decode is the
 * same buffers.  L->events, when set, gets 4 records as in gdn_layer_prefill.  Errors as
 * those calls; y must not overlap the workspace.
 */
gdn_status gdn_layer_decode(const gdn_layer* L, int N, int T, const void* x, long long ldx, float* state,
                            void* conv_state, const int* state_slot, int n_slots, void* y, long long ldy,
                            void* workspace, size_t workspace_bytes, int* err, void* stream);

/*
 * The global-attention layer of the hybrid decoder (the fourth layer of every four):
 * model card "Agnes-3.0-Flash Preview", "Architecture" table, rows "Global attention"
 * and "Positions"; "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model",
 * section "Attention Layer Details".
 * 24 query heads / 4 KV heads of dimension 256, RMS-norm on q and k, rotary position
 * on the first 64 dims of each head (positions = token index within its sequence,
 * base 1e7, pairs (i, i + 32)), causal softmax attention, output * sigmoid(gate).
 * The input projection's output channels: q (24*256) | gate (24*256) | k (4*256) | v (4*256).
 */
#define GDN_ATTN_Q_HEADS 24
#define GDN_ATTN_KV_HEADS 4
#define GDN_ATTN_HEAD_DIM 256
#define GDN_ATTN_N_IN (2 * GDN_ATTN_Q_HEADS * GDN_ATTN_HEAD_DIM + 2 * GDN_ATTN_KV_HEADS * GDN_ATTN_HEAD_DIM)
typedef struct {
  const void* w_in;       /* bf16 [GDN_ATTN_N_IN][ld_w_in], first `hidden` columns used */
  long long ld_w_in;
  const void* w_out;      /* bf16 [hidden][ld_w_out], first 24*256 columns used */
  long long ld_w_out;
  const void* q_norm_w;   /* bf16 [256] */
  const void* k_norm_w;   /* bf16 [256] */
  int hidden;             /* a multiple of 64 */
  void* const* events;    /* optional timing hook: NULL or 4 cudaEvent_t, recorded before the input
                             projection, after it, after the attention, after the output projection */
} gdn_attn_layer;

/*
 * The attention itself, for B sequences of T tokens (packed [B*T]), on given operands:
 *   q_hat  bf16 [B*T][24][256]  normalised, rotated queries
 *   k, v   bf16 [B*T][4][256]   normalised, rotated keys and values (a KV cache)
 *   g      bf16, gate of head h of token t at g + t*ld_g + h*256
 *   out    bf16 [B*T][24*256] = softmax(q_hat k^T / 16, causal within each sequence) v * sigmoid(g),
 *          query head h reading KV head h / 6.
 * The probabilities enter the tensor cores as bf16 (relative error <= 2^-8 each).
 */
gdn_status gdn_attention_prefill(const void* q_hat, const void* k, const void* v, const void* g, long long ld_g,
                                 int B, int T, void* out, int* err, void* stream);

/* Workspace bytes of gdn_attn_layer_prefill for B sequences of T tokens. */
size_t gdn_attn_layer_workspace_size(int B, int T);

/*
 * Prefill of the attention layer for B sequences of T tokens each (packed [B*T]):
 *   x  bf16 [B*T][ldx] -> y bf16 [B*T][ldy] (first `hidden` columns);
 *   k_cache, v_cache  bf16 [B][cache_cap][4][256] (cache_cap = 0: T), rows 0 .. T-1 of each
 *   sequence written: the normalised, rotated keys and the values, i.e. the layer's KV
 *   cache after the prompt (gdn_attn_layer_decode_step continues from it).
 * Launches: gdn_gemm_bf16 (in_proj), the q/k norm + rotary kernel, the flash-attention
 * kernel (tcgen05, gate in its epilogue), gdn_gemm_bf16 (out_proj).  Errors as the
 * other entry points; y, the caches and the workspace must not overlap.  The workspace
 * holds, each from a 1 KiB boundary: the projection [B*T][GDN_ATTN_N_IN], q_hat
 * [B*T][24][256] and the attention output [B*T][24*256] (readable after the call).
 */
gdn_status gdn_attn_layer_prefill(const gdn_attn_layer* L, int B, int T, const void* x, long long ldx,
                                  void* k_cache, void* v_cache, int cache_cap, void* y, long long ldy,
                                  void* workspace, size_t workspace_bytes, int* err, void* stream);

/* Workspace bytes of gdn_attn_layer_decode_step for N sequences with caches of cache_cap rows. */
size_t gdn_attn_decode_workspace_size(int N, int cache_cap);

/*
 * One decode step of the attention layer: one new token per sequence, x bf16 [N][ldx] -> y.
 *   k_cache, v_cache  bf16 [N][cache_cap][4][256]; cache_len  device int32 [N], rows in use,
 *   0 <= cache_len[n] <= cache_cap (a value outside that range is treated like a full cache,
 *   but sets bit 32 of *err instead of 16).
 * The new token's normalised, rotated key and its value go to row cache_len[n] (its rotary
 * position), its queries attend to rows 0 .. cache_len[n], and cache_len[n] grows by one,
 * all on `stream`.  A full cache (cache_len[n] == cache_cap) gives that sequence a zero row of
 * y, leaves its cache and cache_len as they were, and sets bit 16 of *err.  The attention
 * is split over blocks of 512 cache rows and merged exactly; scores and weighted sums are
 * bf16 tensor-core products with fp32 accumulation, the weights entering as a bf16 pair
 * hi + lo (about 16 significant bits), the softmax in fp32.  Workspace: the projection
 * [N][GDN_ATTN_N_IN], q_hat, the attention output [N][24*256] (each from a 1 KiB boundary),
 * then the split partials.
 */
gdn_status gdn_attn_layer_decode_step(const gdn_attn_layer* L, int N, const void* x, long long ldx, void* k_cache,
                                      void* v_cache, int cache_cap, int* cache_len, void* y, long long ldy,
                                      void* workspace, size_t workspace_bytes, int* err, void* stream);

/*
 * T = 1 .. GDN_MAX_DECODE_TOKENS new tokens for each of N sequences in one call
 * (decode with several tokens per step, e.g. verifying drafted tokens), with
 * the states held in slots of a state pool.  Token n * T + t of the inputs is
 * new token t of sequence n (T_tot = N * T); out is bf16 [N * T][H_v][128].
 * The tokens of a sequence are applied in order exactly as T gdn_decode_step
 * calls would apply them (same arithmetic: results are bitwise equal), but each
 * state row is read from HBM once and written once for all T tokens.
 *   state       fp32 [n_slots][H_v][128][128], updated in place
 *   conv_state  bf16 [n_slots][3][C_conv], updated in place (the last 3 raw tokens)
 *   state_slot  device int32 [N]: the slot of sequence n, or NULL for slot n
 *               (then n_slots >= N).  Slots must be distinct within a call.  A slot
 *               outside [0, n_slots) leaves that sequence untouched and sets bit 8
 *               of *err.
 * Inputs must not overlap state, conv_state or out.
 */
#define GDN_MAX_DECODE_TOKENS 8
gdn_status gdn_decode_multi(const gdn_inputs* in, int N, int T, float* state, void* conv_state,
                            const int* state_slot, int n_slots, void* out, int* err, void* stream);

/*
 * Allocation-free prefill.  The pages have no counterpart to this call; it
 * exists for callers that cannot allocate device memory (code running inside a
 * memory budget fixed by a host framework, an allocator hook that must not
 * re-enter the allocator, a runtime whose memory plan is frozen before its
 * first launch).  Same inputs, outputs and results as gdn_prefill, but no
 * workspace argument: the scratch is a file-scope device array of
 * GDN_NOALLOC_SCRATCH_BYTES inside libgdn.so, which every GPU that loads the
 * library holds until the process exits.
 *   - Limit: gdn_prefill_workspace_size(H_k, H_v, B, B*ceil(T/64)) must not
 *     exceed GDN_NOALLOC_SCRATCH_BYTES (64 MiB: e.g. up to 9 chunks of 64
 *     tokens in total at 16/48 heads, 88 at 2/6 heads); larger requests return
 *     GDN_ERR_WORKSPACE and launch nothing.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  The address is kept per device index for
 *     the life of the process: do not use this call across a cudaDeviceReset
 *     (the reset ends the context the address belongs to).
 *   - Every call on a device shares the one array and it keeps the previous
 *     call's contents (nothing in it needs to start at zero).  Calls whose work
 *     overlaps on the GPU -- on different streams, or from different host
 *     threads without ordering -- race on it; order them on one stream.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u << 20)
gdn_status gdn_prefill_noalloc(const gdn_inputs* in, int B, int T, const float* state_in,
                               float* state_out, const void* conv_in, void* conv_out, void* out,
                               int* err, void* stream);

/* Static description of a status code. */
const char* gdn_status_string(gdn_status status);

/*
 * The status that an `err` word (read back after synchronising the stream) stands for:
 * GDN_OK for 0, GDN_ERR_DEVICE_TIMEOUT when bit 1 is set, GDN_ERR_INVALID_ARG for any
 * other bit (device cu_seqlens, a state slot or a KV-cache length the call could not use).
 */
gdn_status gdn_err_status(int err_word);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
