/*
 * hgd_oracle.c -- plain CPU oracle of the hybrid gated-delta decode step.
 *
 * TEST INFRASTRUCTURE ONLY (see hgd_oracle.h).  Single-threaded, no vector
 * intrinsics, built with -O2 -ffp-contract=off and no fast-math, so every sum
 * is evaluated one term at a time in ascending index order, as written.
 * Each routine names the page and section it follows; the abbreviations
 * ([TF], [LUCE], [FT], [AST], [MOE]) are listed in hgd_oracle.h.
 */
#include "hgd_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef hgdo_real real;

/* Elementary functions at the precision of `real`. */
#ifdef HGDO_FP32
#define R_EXP expf
#define R_LOG1P log1pf
#define R_SQRT sqrtf
#define R_FABS fabsf
#else
#define R_EXP exp
#define R_LOG1P log1p
#define R_SQRT sqrt
#define R_FABS fabs
#endif

int hgdo_real_bytes(void) { return (int)sizeof(real); }

/* ------------------------------------------------------------- bf16 ---- */

/* bf16 bit pattern -> value (exact: the upper half of a binary32). */
static inline real bf(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (real)f;
}

real hgdo_bf16_value(uint16_t h) { return bf(h); }

/* Round the exact value to bf16 (8 significant bits, binary32 exponent range),
 * nearest-even.  The quantum at binade 2^(e-1) <= |v| < 2^e is 2^(e-8), and
 * below the smallest normal (2^-126) it is fixed at 2^-133.  v / quantum is
 * exact (a power-of-two scaling in double); nearbyint rounds it half-to-even
 * under the default rounding mode; the product is exact and is a bf16 value,
 * so the conversion to float below is exact too (2^128 becomes +inf). */
static uint16_t round_bf16(real vr) {
    double v = (double)vr;
    if (isnan(v)) return (uint16_t)0x7FC0;
    if (isinf(v)) return v > 0 ? (uint16_t)0x7F80 : (uint16_t)0xFF80;
    if (v == 0.0) return signbit(v) ? (uint16_t)0x8000 : (uint16_t)0x0000;
    int e;
    (void)frexp(v, &e);
    if (e < -125) e = -125;
    double q = ldexp(1.0, e - 8);
    double r = nearbyint(v / q) * q;
    float f = (float)r;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (r == 0.0) u = signbit(v) ? 0x80000000u : 0u;
    return (uint16_t)(u >> 16);
}

uint16_t hgdo_round_bf16(real v) { return round_bf16(v); }

void hgdo_round_bf16_array(const real* v, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(v[i]);
}

/* ------------------------------------------------------- scalar maps --- */

static real silu(real t) { return t / ((real)1 + R_EXP(-t)); }
static real sigmoid(real t) { return (real)1 / ((real)1 + R_EXP(-t)); }
/* [MOE] activation_topk: max(x,0) + log1p(exp(-|x|)). */
static real softplus(real t) { return (t > 0 ? t : (real)0) + R_LOG1P(R_EXP(-R_FABS(t))); }

real hgdo_softplus(real t) { return softplus(t); }

/* Log-decay of the GDN layers of the stack, one per head ([TF] PR body: the
 * gated delta rule; commit on config.json widths: A_log stored as bf16):
 *   g[h] = -exp(A_log[h]) * softplus(a[h] + dt_bias[h]),  so alpha = exp(g) in (0, 1]. */
void hgdo_gdn_gates(const real* a, const uint16_t* A_log, const uint16_t* dt_bias, real* g, int H) {
    for (int h = 0; h < H; ++h) g[h] = -R_EXP(bf(A_log[h])) * softplus(a[h] + bf(dt_bias[h]));
}

/* ------------------------------------------------------------ GEMV ----- */

/* [AST] BF16 GEMV: y = x W^T with W in the [N,K] (Linear) layout.  (In the
 * all-cores build the output elements are shared out over threads; each one's
 * sum runs in the same order, so the results do not change.) */
void hgdo_gemv(const uint16_t* W, const uint16_t* x, real* y, int M, int N, int K) {
    for (int m = 0; m < M; ++m) {
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            real s = 0;
            for (int k = 0; k < K; ++k)
                s += bf(W[(int64_t)n * K + k]) * bf(x[(int64_t)m * K + k]);
            y[(int64_t)m * N + n] = s;
        }
    }
}

/* [AST] fused up/gate SwiGLU, [FT] silu_and_mul: bf16(silu(g) * u). */
void hgdo_swiglu(const uint16_t* Wg, const uint16_t* Wu, const uint16_t* x, uint16_t* h,
                 int M, int I, int K) {
    real* g = (real*)malloc(sizeof(real) * (size_t)M * I);
    real* u = (real*)malloc(sizeof(real) * (size_t)M * I);
    hgdo_gemv(Wg, x, g, M, I, K);
    hgdo_gemv(Wu, x, u, M, I, K);
    for (int64_t i = 0; i < (int64_t)M * I; ++i) h[i] = round_bf16(silu(g[i]) * u[i]);
    free(g);
    free(u);
}

/* ------------------------------------------------------------ conv ----- */

/* [TF] causal convolution with a per-stream tail, recorded per row. */
void hgdo_conv1d_tail_update(const real* x, real* tail, const uint16_t* w, real* y,
                             real* tail_rec, int B, int T, int C, int kc, int apply_silu) {
    const int nt = kc - 1;
    for (int b = 0; b < B; ++b) {
        real* tb = tail + (int64_t)b * nt * C;
        for (int t = 0; t < T; ++t) {
            const real* xr = x + ((int64_t)b * T + t) * C;
            real* yr = y + ((int64_t)b * T + t) * C;
            for (int c = 0; c < C; ++c) {
                real s = 0;
                for (int j = 0; j < nt; ++j) s += bf(w[(int64_t)c * kc + j]) * tb[(int64_t)j * C + c];
                s += bf(w[(int64_t)c * kc + nt]) * xr[c];
                yr[c] = apply_silu ? silu(s) : s;
            }
            for (int c = 0; c < C; ++c) {
                for (int j = 0; j + 1 < nt; ++j) tb[(int64_t)j * C + c] = tb[(int64_t)(j + 1) * C + c];
                if (nt > 0) tb[(int64_t)(nt - 1) * C + c] = xr[c];
            }
            if (tail_rec)
                memcpy(tail_rec + ((int64_t)b * T + t) * nt * C, tb, sizeof(real) * (size_t)nt * C);
        }
    }
}

/* ------------------------------------------------------ gated delta ---- */

static void l2normalize(real* v, int n) {
    real ss = 0;
    for (int i = 0; i < n; ++i) ss += v[i] * v[i];
    real inv = (real)1 / R_SQRT(ss + (real)1e-6);
    for (int i = 0; i < n; ++i) v[i] = v[i] * inv;
}

/* One head, one row: the dense form of the gated delta rule. */
static void gdn_head_row(real* S, const real* q_in, const real* k_in, const real* v,
                         real g, real braw, real* o, int dk, int dv, int l2norm,
                         real* qn, real* kn, real* A, real* Snew) {
    for (int i = 0; i < dk; ++i) { qn[i] = q_in[i]; kn[i] = k_in[i]; }
    if (l2norm) { l2normalize(qn, dk); l2normalize(kn, dk); }
    const real alpha = R_EXP(g);
    const real beta = sigmoid(braw);
    /* A = I - beta k k^T */
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dk; ++j)
            A[(int64_t)i * dk + j] = (i == j ? (real)1 : (real)0) - beta * (kn[i] * kn[j]);
    /* S A: element (i,j) is sum_l S[i][l] A[l][j], summed over ascending l
     * (the l-loop is outside the j-loop only so that A is read row by row). */
    for (int64_t n = 0; n < (int64_t)dv * dk; ++n) Snew[n] = 0;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < dv; ++i)
        for (int l = 0; l < dk; ++l) {
            const real s_il = S[(int64_t)i * dk + l];
            for (int j = 0; j < dk; ++j) Snew[(int64_t)i * dk + j] += s_il * A[(int64_t)l * dk + j];
        }
    /* S <- alpha (S A) + beta v k^T */
    for (int i = 0; i < dv; ++i)
        for (int j = 0; j < dk; ++j)
            S[(int64_t)i * dk + j] = alpha * Snew[(int64_t)i * dk + j] + beta * (v[i] * kn[j]);
    /* o = S q with the updated S */
    for (int i = 0; i < dv; ++i) {
        real s = 0;
        for (int j = 0; j < dk; ++j) s += S[(int64_t)i * dk + j] * qn[j];
        o[i] = s;
    }
}

/* [TF] commit on the widths read from config.json: linear (GDN) value heads over
 * fewer key heads.  Value head h reads query/key head h / (Hv / Hk); the gates,
 * the value, the state and the output are per value head. */
void hgdo_gdn_step_grouped(const real* q, const real* k, const real* v, int64_t row_stride,
                           const real* g, const real* braw, real* S, real* o, real* S_rec,
                           int B, int T, int Hk, int H, int dk, int dv, int l2norm) {
    const int grp = H / Hk;
    real* qn = (real*)malloc(sizeof(real) * (size_t)dk);
    real* kn = (real*)malloc(sizeof(real) * (size_t)dk);
    real* A = (real*)malloc(sizeof(real) * (size_t)dk * dk);
    real* Snew = (real*)malloc(sizeof(real) * (size_t)dv * dk);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            const int64_t row = (int64_t)b * T + t;
            for (int h = 0; h < H; ++h) {
                real* Sh = S + ((int64_t)b * H + h) * dv * dk;
                gdn_head_row(Sh, q + row * row_stride + (int64_t)(h / grp) * dk,
                             k + row * row_stride + (int64_t)(h / grp) * dk,
                             v + row * row_stride + (int64_t)h * dv,
                             g[row * H + h], braw[row * H + h],
                             o + (row * H + h) * dv, dk, dv, l2norm, qn, kn, A, Snew);
                if (S_rec)
                    memcpy(S_rec + (row * H + h) * dv * dk, Sh, sizeof(real) * (size_t)dv * dk);
            }
        }
    free(qn); free(kn); free(A); free(Snew);
}

void hgdo_gdn_step(const real* q, const real* k, const real* v, int64_t row_stride,
                   const real* g, const real* braw, real* S, real* o, real* S_rec,
                   int B, int T, int H, int dk, int dv, int l2norm) {
    hgdo_gdn_step_grouped(q, k, v, row_stride, g, braw, S, o, S_rec, B, T, H, H, dk, dv, l2norm);
}

/* ------------------------------------------ recurrence logs and keep ---- */
/* [TF] tree-window commit note: a verify window no longer snapshots every row's
 * state; each stream logs its rows' decay, write and key, and keep replays the
 * kept rows onto the recurrence in one pass.  Written out: the update of row t
 *   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 * equals  alpha_t S_{t-1} + delta_t k_t^T  with the write
 *   delta_t = beta_t (v_t - alpha_t S_{t-1} k_t),
 * so (alpha_t, delta_t, k_t) determine S_t from S_{t-1} without v, beta or q. */

void hgdo_gdn_window_log(const real* q, const real* k, const real* v, int64_t row_stride,
                         const real* g, const real* braw, const real* S, real* o,
                         real* log_alpha, real* log_delta, real* log_k,
                         int B, int T, int H, int dk, int dv, int l2norm) {
    real* qn = (real*)malloc(sizeof(real) * (size_t)dk);
    real* kn = (real*)malloc(sizeof(real) * (size_t)dk);
    real* A = (real*)malloc(sizeof(real) * (size_t)dk * dk);
    real* Snew = (real*)malloc(sizeof(real) * (size_t)dv * dk);
    real* Sw = (real*)malloc(sizeof(real) * (size_t)dv * dk);   /* the window's running state */
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            memcpy(Sw, S + ((int64_t)b * H + h) * dv * dk, sizeof(real) * (size_t)dv * dk);
            for (int t = 0; t < T; ++t) {
                const int64_t row = (int64_t)b * T + t;
                const real* kr = k + row * row_stride + (int64_t)h * dk;
                const real* vr = v + row * row_stride + (int64_t)h * dv;
                const real alpha = R_EXP(g[row * H + h]);
                const real beta = sigmoid(braw[row * H + h]);
                /* the logged key: k, L2-normalised as the step normalises it */
                real* lk = log_k + (row * H + h) * dk;
                for (int i = 0; i < dk; ++i) lk[i] = kr[i];
                if (l2norm) l2normalize(lk, dk);
                /* the write, from the state before the row */
                real* ld = log_delta + (row * H + h) * dv;
                for (int i = 0; i < dv; ++i) {
                    real w = 0;
                    for (int j = 0; j < dk; ++j) w += Sw[(int64_t)i * dk + j] * lk[j];
                    ld[i] = beta * (vr[i] - alpha * w);
                }
                log_alpha[row * H + h] = alpha;
                /* the row itself, as hgdo_gdn_step computes it, on the running copy */
                gdn_head_row(Sw, q + row * row_stride + (int64_t)h * dk, kr, vr, g[row * H + h],
                             braw[row * H + h], o + (row * H + h) * dv, dk, dv, l2norm, qn, kn, A, Snew);
            }
        }
    free(qn); free(kn); free(A); free(Snew); free(Sw);
}

int hgdo_gdn_keep(real* S, const real* log_alpha, const real* log_delta, const real* log_k,
                  const int32_t* keep, int B, int T, int H, int dk, int dv) {
    for (int b = 0; b < B; ++b)
        if (keep[b] < 0 || keep[b] > T) return 2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            real* Sh = S + ((int64_t)b * H + h) * dv * dk;
            for (int t = 0; t < keep[b]; ++t) {
                const int64_t lr = ((int64_t)b * T + t) * H + h;
                const real alpha = log_alpha[lr];
                const real* dl = log_delta + lr * dv;
                const real* kk = log_k + lr * dk;
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j)
                        Sh[(int64_t)i * dk + j] = alpha * Sh[(int64_t)i * dk + j] + dl[i] * kk[j];
            }
        }
    return 0;
}

/* The conv tail after the first keep[b] rows of a window whose inputs are x
 * [B][T][C]: the newest kc-1 entries of (tail, x_0, ..., x_{keep-1}). */
int hgdo_conv1d_keep(real* tail, const real* x, const int32_t* keep, int B, int T, int C, int kc) {
    const int nt = kc - 1;
    for (int b = 0; b < B; ++b)
        if (keep[b] < 0 || keep[b] > T) return 2;
    for (int b = 0; b < B; ++b) {
        real* tb = tail + (int64_t)b * nt * C;
        for (int t = 0; t < keep[b]; ++t) {
            const real* xr = x + ((int64_t)b * T + t) * C;
            for (int c = 0; c < C; ++c) {
                for (int j = 0; j + 1 < nt; ++j) tb[(int64_t)j * C + c] = tb[(int64_t)(j + 1) * C + c];
                if (nt > 0) tb[(int64_t)(nt - 1) * C + c] = xr[c];
            }
        }
    }
    return 0;
}

/* ----------------------------------------------------------- norms ----- */

/* [FT] RMSNorm. */
void hgdo_rmsnorm(const uint16_t* x, const uint16_t* w, uint16_t* y, int M, int D, double eps) {
    for (int m = 0; m < M; ++m) {
        const uint16_t* xr = x + (int64_t)m * D;
        real ss = 0;
        for (int i = 0; i < D; ++i) ss += bf(xr[i]) * bf(xr[i]);
        real r = (real)1 / R_SQRT(ss / (real)D + (real)eps);
        for (int i = 0; i < D; ++i) y[(int64_t)m * D + i] = round_bf16(bf(xr[i]) * r * bf(w[i]));
    }
}

/* [FT] gated RMSNorm, per head over d. */
void hgdo_gated_rmsnorm(const real* o, const uint16_t* z, const uint16_t* w, uint16_t* u,
                        int M, int nh, int d, double eps) {
    for (int m = 0; m < M; ++m)
        for (int h = 0; h < nh; ++h) {
            const int64_t base = (int64_t)m * nh * d + (int64_t)h * d;
            real ss = 0;
            for (int i = 0; i < d; ++i) ss += o[base + i] * o[base + i];
            real r = (real)1 / R_SQRT(ss / (real)d + (real)eps);
            for (int i = 0; i < d; ++i)
                u[base + i] = round_bf16(o[base + i] * r * bf(w[i]) * silu(bf(z[base + i])));
        }
}

/* ------------------------------------------------------- attention ----- */

void hgdo_rope(real* x, int hd, int pos, double base) {
    const int half = hd / 2;
    for (int i = 0; i < half; ++i) {
        double th = (double)pos * pow(base, -2.0 * (double)i / (double)hd);
        real c = (real)cos(th), s = (real)sin(th);
        real a = x[i], b = x[i + half];
        x[i] = a * c - b * s;
        x[i + half] = b * c + a * s;
    }
}

/* [TF] gated attention for one decode row. */
void hgdo_attention_row(const real* q, const real* gate, const uint16_t* Kc, const uint16_t* Vc,
                        int nkeys, int Lmax, int nq, int nkv, int hd, uint16_t* out) {
    const int group = nq / nkv;
    const real scale = (real)1 / R_SQRT((real)hd);
    real* s = (real*)malloc(sizeof(real) * (size_t)(nkeys > 0 ? nkeys : 1));
    for (int i = 0; i < nq; ++i) {
        const int g = i / group;
        const uint16_t* K = Kc + (int64_t)g * Lmax * hd;
        const uint16_t* V = Vc + (int64_t)g * Lmax * hd;
        const real* qi = q + (int64_t)i * hd;
        real mx = -INFINITY;
        for (int j = 0; j < nkeys; ++j) {
            real d = 0;
            for (int e = 0; e < hd; ++e) d += qi[e] * bf(K[(int64_t)j * hd + e]);
            s[j] = d * scale;
            if (s[j] > mx) mx = s[j];
        }
        real l = 0;
        for (int j = 0; j < nkeys; ++j) { s[j] = R_EXP(s[j] - mx); l += s[j]; }
        for (int e = 0; e < hd; ++e) {
            real acc = 0;
            for (int j = 0; j < nkeys; ++j) acc += (s[j] / l) * bf(V[(int64_t)j * hd + e]);
            out[(int64_t)i * hd + e] = round_bf16(acc * sigmoid(gate[(int64_t)i * hd + e]));
        }
    }
    free(s);
}

/* ----------------------------------------------------------- stack ----- */

static int is_attn(const hgdo_config* c, int l) { return (l % c->attn_every) == c->attn_every - 1; }

static void add_residual(uint16_t* x, const real* delta, int D) {
    for (int i = 0; i < D; ++i) x[i] = round_bf16(bf(x[i]) + delta[i]);
}

int hgdo_decode_stack(const hgdo_model* m, hgdo_state* st, const int32_t* tokens, int T,
                      real* logits, int32_t* argmax, real* S_rec, real* tail_rec, uint16_t* x_rec) {
    const hgdo_config* c = &m->cfg;
    const int L = c->n_layers, D = c->hidden, V = c->vocab, Hk = c->gdn_heads;
    const int H = c->gdn_v_heads > 0 ? c->gdn_v_heads : Hk;  /* value heads */
    const int dk = c->gdn_dk, dv = c->gdn_dv, kc = c->conv_k, nq = c->attn_q_heads;
    const int nkv = c->attn_kv_heads, hd = c->attn_head_dim, I = c->mlp_inter;
    const int B = st->B, Lmax = st->Lmax;
    const int Cc = 2 * Hk * dk + H * dv;              /* conv channels q|k|v */
    const int n_gdn_out = Cc + H * dv + 2 * H;        /* q|k|v|z|a|b */
    const int n_att_out = 2 * nq * hd + 2 * nkv * hd; /* q|gate|k|v */
    if (L > HGDO_MAX_LAYERS || L <= 0 || H % Hk != 0) return 2;
    int n_gdn = 0, n_attn = 0;
    for (int l = 0; l < L; ++l) { if (is_attn(c, l)) ++n_attn; else ++n_gdn; }
    for (int b = 0; b < B; ++b) {
        if (st->pos[b] < 0 || st->pos[b] + T > Lmax) return 2;
        for (int t = 0; t < T; ++t)
            if (tokens[b * T + t] < 0 || tokens[b * T + t] >= V) return 2;
    }

    const int wmax = n_gdn_out > n_att_out ? n_gdn_out : n_att_out;
    uint16_t* x = (uint16_t*)malloc(sizeof(uint16_t) * D);
    uint16_t* h = (uint16_t*)malloc(sizeof(uint16_t) * D);
    real* p = (real*)malloc(sizeof(real) * wmax);
    real* y = (real*)malloc(sizeof(real) * Cc);
    real* o = (real*)malloc(sizeof(real) * (size_t)(H * dv > nq * hd ? H * dv : nq * hd));
    uint16_t* z = (uint16_t*)malloc(sizeof(uint16_t) * H * dv);
    uint16_t* u = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(H * dv > nq * hd ? H * dv : nq * hd));
    real* gg = (real*)malloc(sizeof(real) * H);
    real* bb = (real*)malloc(sizeof(real) * H);
    real* dlt = (real*)malloc(sizeof(real) * D);
    uint16_t* mm = (uint16_t*)malloc(sizeof(uint16_t) * I);
    real* lg = (real*)malloc(sizeof(real) * V);
    int status = 0;

    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            const int row = b * T + t;
            const int P = st->pos[b] + t;
            memcpy(x, m->embed + (int64_t)tokens[row] * D, sizeof(uint16_t) * D);
            int ig = 0, ia = 0;
            for (int l = 0; l < L; ++l) {
                const hgdo_layer* w = &m->layers[l];
                hgdo_rmsnorm(x, w->in_norm, h, 1, D, c->norm_eps);
                if (!is_attn(c, l)) {
                    hgdo_gemv(w->w_in, h, p, 1, n_gdn_out, D);
                    real* S = st->S + ((int64_t)ig * B + b) * H * dv * dk;
                    real* tl = st->tail + ((int64_t)ig * B + b) * (kc - 1) * Cc;
                    real* trec = tail_rec ? tail_rec + (((int64_t)ig * B + b) * T + t) * (kc - 1) * Cc : NULL;
                    hgdo_conv1d_tail_update(p, tl, w->conv_w, y, trec, 1, 1, Cc, kc, 1);
                    for (int i = 0; i < H * dv; ++i) z[i] = round_bf16(p[Cc + i]);
                    hgdo_gdn_gates(p + Cc + H * dv, w->A_log, w->dt_bias, gg, H);
                    for (int hh = 0; hh < H; ++hh) bb[hh] = p[Cc + H * dv + H + hh];
                    real* srec = S_rec ? S_rec + (((int64_t)ig * B + b) * T + t) * H * dv * dk : NULL;
                    hgdo_gdn_step_grouped(y, y + Hk * dk, y + 2 * Hk * dk, Cc, gg, bb, S, o, srec,
                                          1, 1, Hk, H, dk, dv, 1);
                    hgdo_gated_rmsnorm(o, z, w->gnorm_w, u, 1, H, dv, c->norm_eps);
                    hgdo_gemv(w->w_out, u, dlt, 1, D, H * dv);
                    add_residual(x, dlt, D);
                    ++ig;
                } else {
                    hgdo_gemv(w->w_in, h, p, 1, n_att_out, D);
                    real* qr = p;
                    real* gate = p + nq * hd;
                    real* kr = p + 2 * nq * hd;
                    real* vr = p + 2 * nq * hd + nkv * hd;
                    for (int i = 0; i < nq; ++i) hgdo_rope(qr + (int64_t)i * hd, hd, P, c->rope_base);
                    for (int g = 0; g < nkv; ++g) hgdo_rope(kr + (int64_t)g * hd, hd, P, c->rope_base);
                    uint16_t* Kc = st->kv + (((int64_t)ia * 2 + 0) * B + b) * nkv * Lmax * hd;
                    uint16_t* Vc = st->kv + (((int64_t)ia * 2 + 1) * B + b) * nkv * Lmax * hd;
                    for (int g = 0; g < nkv; ++g)
                        for (int e = 0; e < hd; ++e) {
                            Kc[((int64_t)g * Lmax + P) * hd + e] = round_bf16(kr[g * hd + e]);
                            Vc[((int64_t)g * Lmax + P) * hd + e] = round_bf16(vr[g * hd + e]);
                        }
                    hgdo_attention_row(qr, gate, Kc, Vc, P + 1, Lmax, nq, nkv, hd, u);
                    hgdo_gemv(w->w_out, u, dlt, 1, D, nq * hd);
                    add_residual(x, dlt, D);
                    ++ia;
                }
                hgdo_rmsnorm(x, w->post_norm, h, 1, D, c->norm_eps);
                hgdo_swiglu(w->w_gate, w->w_up, h, mm, 1, I, D);
                hgdo_gemv(w->w_down, mm, dlt, 1, D, I);
                add_residual(x, dlt, D);
                if (x_rec) memcpy(x_rec + (((int64_t)l * B + b) * T + t) * D, x, sizeof(uint16_t) * D);
            }
            hgdo_rmsnorm(x, m->final_norm, h, 1, D, c->norm_eps);
            hgdo_gemv(m->lm_head ? m->lm_head : m->embed, h, lg, 1, V, D);
            /* [MOE] top-k: on equal scores the lower index wins; the decision is
             * taken on the logits as binary32 values. */
            int best = -1;
            float bv = 0.0f;
            for (int j = 0; j < V; ++j) {
                float f = (float)lg[j];
                if (isnan(f)) { best = -1; status = 1; break; }
                if (best < 0 || f > bv) { best = j; bv = f; }
            }
            argmax[row] = best;
            if (logits) memcpy(logits + (int64_t)row * V, lg, sizeof(real) * (size_t)V);
        }
    }
    for (int b = 0; b < B; ++b) st->pos[b] += T;
    free(x); free(h); free(p); free(y); free(o); free(z); free(u);
    free(gg); free(bb); free(dlt); free(mm); free(lg);
    return status;
}
