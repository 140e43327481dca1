/*
 * Oracle for the gated-delta-rule token mixer -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * this library.  The CUDA product path never links, loads or calls it, and this
 * file shares no code, header, table or constant with it.
 *
 * What it computes (plain fp64, one token at a time, in the order the method
 * states it):
 *   Agnes-3.0-Flash model card, "Architecture" table, row "Delta-rule layers":
 *     16 key heads / 48 value heads, head dim 128, a causal conv of kernel 4 in
 *     front, a gated RMS-norm after, recurrent state in fp32.
 *   "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention Multimodal Model",
 *     section "Feed-Forward and Positional Encoding", paragraph on the Gated
 *     Delta Rule: each step first erases the old association of the key and
 *     then writes the new value ("erase then update"), and a forget gate
 *     decays the whole memory.
 *   The recurrence those two passages name, written out (the standard gated
 *   delta rule; the pages give no equation, so this is the reading taken):
 *       S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t
 *   with S_t a d_v x d_k matrix per value head.
 *
 * Readings of points the pages leave open:
 *   - conv: depthwise over the q|k|v channels, no bias, tap 3 on the current
 *     token, history before a sequence start from conv_in (zeros if absent);
 *     SiLU after the conv.
 *   - q and k are L2-normalised per head as x / sqrt(sum x^2 + 1e-6); q is then
 *     multiplied by `scale` (1.0 by default).
 *   - gates: g = -exp(A_log[h]) * softplus(a), alpha = exp(g), beta = sigmoid(b).
 *   - value head h reads key head h / (H_v / H_k) (contiguous groups).
 *   - gated RMS-norm per value head over d_v:
 *       y = o / sqrt(mean(o^2) + 1e-6) * w * SiLU(z).
 *
 * Every input arrives as the exact bf16/fp32 value the GPU sees and is widened
 * to fp64; all arithmetic below is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_TAPS 4
#define ORACLE_EPS 1e-6

static double bf16_value(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double silu(double y) { return y / (1.0 + exp(-y)); }

static double softplus(double a) {
    if (a > 30.0) return a + log1p(exp(-a));
    return log1p(exp(a));
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ---- stage helpers (one token / one row) -------------------------------- */

/* Causal depthwise conv of one channel: window[i] is x(t - 3 + i). */
static double conv_window(const double* window, const double* w4) {
    double acc = 0.0;
    for (int i = 0; i < ORACLE_TAPS; ++i) acc += w4[i] * window[i];
    return acc;
}

/* x <- x / sqrt(sum x^2 + eps) */
static void l2norm_row(double* x, int n) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss + ORACLE_EPS);
    for (int i = 0; i < n; ++i) x[i] *= inv;
}

/* One step of the gated delta rule for one value head (S is dv x dk, row-major):
 *   S <- alpha S;  p = S k;  S <- S + beta (v - p) k^T;  o = S q.
 * This is S_t = alpha S_{t-1}(I - beta k k^T) + beta v k^T, o_t = S_t q_t. */
static void delta_step(double* S, int dv, int dk, const double* q, const double* k,
                       const double* v, double alpha, double beta, double* o) {
    for (int r = 0; r < dv; ++r) {
        double* s = S + (size_t)r * dk;
        double p = 0.0;
        for (int c = 0; c < dk; ++c) {
            s[c] *= alpha;
            p += s[c] * k[c];
        }
        double delta = beta * (v[r] - p);
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) {
            s[c] += delta * k[c];
            acc += s[c] * q[c];
        }
        o[r] = acc;
    }
}

/* y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) */
static void gated_rmsnorm_row(const double* o, const double* z, const double* w, int n, double* y) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += o[i] * o[i];
    double inv = 1.0 / sqrt(ss / n + ORACLE_EPS);
    for (int i = 0; i < n; ++i) y[i] = o[i] * inv * w[i] * silu(z[i]);
}

/* ---- exported stage functions (used by the pins) ------------------------ */

/* y[t][c] = SiLU?( sum_i w[c][i] x[t-3+i][c] ) per sequence; rows before a
 * sequence start come from hist[n][0..2][c] (oldest first) or are zero. */
void gdn_oracle_conv(int n_seq, const int64_t* cu_seqlens, int C, const double* x,
                     const double* w, const double* hist, int apply_silu, double* y) {
    for (int n = 0; n < n_seq; ++n) {
        int64_t s = cu_seqlens[n], e = cu_seqlens[n + 1];
        for (int64_t t = s; t < e; ++t) {
            for (int c = 0; c < C; ++c) {
                double win[ORACLE_TAPS];
                for (int i = 0; i < ORACLE_TAPS; ++i) {
                    int64_t tau = t - (ORACLE_TAPS - 1) + i;
                    if (tau >= s) win[i] = x[(size_t)tau * C + c];
                    else if (hist) win[i] = hist[((size_t)n * 3 + (size_t)(3 + (tau - s))) * C + c];
                    else win[i] = 0.0;
                }
                double v = conv_window(win, w + (size_t)c * ORACLE_TAPS);
                y[(size_t)t * C + c] = apply_silu ? silu(v) : v;
            }
        }
    }
}

void gdn_oracle_l2norm(int64_t rows, int n, const double* x, double* y) {
    for (int64_t r = 0; r < rows; ++r) {
        memcpy(y + r * n, x + r * n, sizeof(double) * (size_t)n);
        l2norm_row(y + r * n, n);
    }
}

/* g = -exp(A_log[h]) softplus(a[t][h]); alpha = exp(g); beta = sigmoid(b) */
void gdn_oracle_gates(int64_t T, int H, const double* A_log, const double* a, const double* b,
                      double* g, double* alpha, double* beta) {
    for (int64_t t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            size_t i = (size_t)t * H + h;
            double gg = -exp(A_log[h]) * softplus(a[i]);
            if (g) g[i] = gg;
            alpha[i] = exp(gg);
            beta[i] = sigmoid(b[i]);
        }
}

/* The recurrence alone on post-front-end q,k ([T][H_k][dk]), v ([T][H_v][dv]),
 * alpha, beta ([T][H_v]).  S0: [n_seq][H_v][dv][dk] or NULL (zeros).
 * o: [T][H_v][dv] (pre-norm).  S_out: [n_seq][H_v][dv][dk] or NULL. */
void gdn_oracle_recurrence(int n_seq, const int64_t* cu_seqlens, int H_k, int H_v, int dk, int dv,
                           const double* q, const double* k, const double* v,
                           const double* alpha, const double* beta, const double* S0,
                           double* o, double* S_out) {
    int G = H_v / H_k;
    double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
    for (int n = 0; n < n_seq; ++n)
        for (int h = 0; h < H_v; ++h) {
            size_t soff = ((size_t)n * H_v + h) * (size_t)dv * dk;
            if (S0) memcpy(S, S0 + soff, sizeof(double) * (size_t)dv * dk);
            else memset(S, 0, sizeof(double) * (size_t)dv * dk);
            int kh = h / G;
            for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
                size_t gi = (size_t)t * H_v + h;
                delta_step(S, dv, dk, q + ((size_t)t * H_k + kh) * dk, k + ((size_t)t * H_k + kh) * dk,
                           v + gi * dv, alpha[gi], beta[gi], o + gi * dv);
            }
            if (S_out) memcpy(S_out + soff, S, sizeof(double) * (size_t)dv * dk);
        }
    free(S);
}

void gdn_oracle_gated_rmsnorm(int64_t rows, int n, const double* o, const double* z,
                              const double* w, double* y) {
    for (int64_t r = 0; r < rows; ++r) gated_rmsnorm_row(o + r * n, z + r * n, w, n, y + r * n);
}

/* ---- the whole mixer, streamed per (sequence, value head) ---------------- */

typedef struct {
    int n_seq;
    const int64_t* cu;
    int H_k, H_v, D, C_conv;
    const uint16_t *q, *k, *v, *a, *b, *z, *conv_w, *norm_w;
    const float* A_log;
    double scale;
    const float* state_in;
    const uint16_t* conv_in;
} oracle_args;

/* raw value of conv channel c at token tau of sequence n (history if before start) */
static double raw_channel(const oracle_args* A, int n, int64_t tau, int c) {
    int64_t s = A->cu[n];
    if (tau >= s) {
        int qk = A->H_k * A->D;
        if (c < qk) return bf16_value(A->q[(size_t)tau * qk + c]);
        if (c < 2 * qk) return bf16_value(A->k[(size_t)tau * qk + (c - qk)]);
        return bf16_value(A->v[(size_t)tau * (size_t)(A->H_v * A->D) + (c - 2 * qk)]);
    }
    if (!A->conv_in) return 0.0;
    return bf16_value(A->conv_in[((size_t)n * 3 + (size_t)(3 + (tau - s))) * A->C_conv + c]);
}

/* conv + SiLU of channels [c0, c0+len) at token t of sequence n */
static void front_channels(const oracle_args* A, int n, int64_t t, int c0, int len, double* out) {
    for (int j = 0; j < len; ++j) {
        int c = c0 + j;
        double win[ORACLE_TAPS], w4[ORACLE_TAPS];
        for (int i = 0; i < ORACLE_TAPS; ++i) {
            win[i] = raw_channel(A, n, t - (ORACLE_TAPS - 1) + i, c);
            w4[i] = bf16_value(A->conv_w[(size_t)c * ORACLE_TAPS + i]);
        }
        out[j] = silu(conv_window(win, w4));
    }
}

static void mixer_task(const oracle_args* A, int n, int h, double* out, double* state_out,
                       double* pre_norm) {
    int D = A->D, G = A->H_v / A->H_k, kh = h / G;
    int qk = A->H_k * D;
    double* S = (double*)malloc(sizeof(double) * (size_t)D * D);
    double* buf = (double*)malloc(sizeof(double) * (size_t)D * 7);
    double *q = buf, *k = buf + D, *v = buf + 2 * D, *o = buf + 3 * D, *z = buf + 4 * D,
           *w = buf + 5 * D, *y = buf + 6 * D;
    size_t soff = ((size_t)n * A->H_v + h) * (size_t)D * D;
    for (size_t i = 0; i < (size_t)D * D; ++i) S[i] = A->state_in ? (double)A->state_in[soff + i] : 0.0;
    for (int i = 0; i < D; ++i) w[i] = bf16_value(A->norm_w[i]);
    double decay_scale = exp((double)A->A_log[h]);
    for (int64_t t = A->cu[n]; t < A->cu[n + 1]; ++t) {
        front_channels(A, n, t, kh * D, D, q);
        front_channels(A, n, t, qk + kh * D, D, k);
        front_channels(A, n, t, 2 * qk + h * D, D, v);
        l2norm_row(q, D);
        l2norm_row(k, D);
        for (int i = 0; i < D; ++i) q[i] *= A->scale;
        size_t gi = (size_t)t * A->H_v + h;
        double g = -decay_scale * softplus(bf16_value(A->a[gi]));
        double alpha = exp(g), beta = sigmoid(bf16_value(A->b[gi]));
        delta_step(S, D, D, q, k, v, alpha, beta, o);
        for (int i = 0; i < D; ++i) z[i] = bf16_value(A->z[gi * D + i]);
        gated_rmsnorm_row(o, z, w, D, y);
        if (out) memcpy(out + gi * D, y, sizeof(double) * (size_t)D);
        if (pre_norm) memcpy(pre_norm + gi * D, o, sizeof(double) * (size_t)D);
    }
    if (state_out) memcpy(state_out + soff, S, sizeof(double) * (size_t)D * D);
    free(buf);
    free(S);
}

/*
 * Full mixer over a packed batch of sequences (cu_seqlens int64 [n_seq+1]).
 *   q, k: bf16 bits [T_tot][H_k][D]; v, z: [T_tot][H_v][D]; a, b: [T_tot][H_v]
 *   conv_w: bf16 [C_conv][4] with C_conv = (2 H_k + H_v) D, channels q|k|v
 *   A_log: fp32 [H_v]; norm_w: bf16 [D]
 *   state_in: fp32 [n_seq][H_v][D][D] or NULL; conv_in: bf16 [n_seq][3][C_conv] or NULL
 *   heads: value heads to compute (NULL = all); only those heads' out / state_out
 *   / pre_norm entries are written.
 *   out: fp64 [T_tot][H_v][D]; state_out: fp64 [n_seq][H_v][D][D] or NULL;
 *   conv_out: fp64 [n_seq][3][C_conv] or NULL (all channels); pre_norm: fp64
 *   [T_tot][H_v][D] or NULL (o_t before the gated norm).
 * Returns 0, or -1 on a bad argument.
 */
int gdn_oracle_mixer(int n_seq, const int64_t* cu_seqlens, int H_k, int H_v, int D,
                     const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* a,
                     const uint16_t* b, const uint16_t* z, const uint16_t* conv_w,
                     const float* A_log, const uint16_t* norm_w, double scale,
                     const float* state_in, const uint16_t* conv_in, const int* heads, int n_heads,
                     double* out, double* state_out, double* conv_out, double* pre_norm,
                     int n_threads) {
    if (n_seq < 0 || H_k <= 0 || H_v <= 0 || D <= 0 || H_v % H_k != 0) return -1;
    for (int n = 0; n < n_seq; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    oracle_args A = {n_seq, cu_seqlens, H_k, H_v, D, (2 * H_k + H_v) * D, q, k, v, a, b, z,
                     conv_w, norm_w, A_log, scale, state_in, conv_in};
    int nh = heads ? n_heads : H_v;
    long long tasks = (long long)n_seq * nh;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long i = 0; i < tasks; ++i) {
        int n = (int)(i / nh);
        int h = heads ? heads[i % nh] : (int)(i % nh);
        mixer_task(&A, n, h, out, state_out, pre_norm);
    }
    if (conv_out) {
        for (int n = 0; n < n_seq; ++n) {
            int64_t e = cu_seqlens[n + 1];
            for (int j = 0; j < 3; ++j)
                for (int c = 0; c < A.C_conv; ++c)
                    conv_out[((size_t)n * 3 + j) * A.C_conv + c] = raw_channel(&A, n, e - 3 + j, c);
        }
    }
    return 0;
}

int gdn_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
