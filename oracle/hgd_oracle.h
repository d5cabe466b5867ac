/*
 * hgd_oracle.h -- plain, slow CPU oracle of the hybrid gated-delta decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this library: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no source with the CUDA library (no headers, helpers,
 * tables or constants) and follows the method as written, one loop per sum,
 * in ascending index order, with no blocking, fusion or algebraic rewrite.
 *
 * Arithmetic type.  Every floating-point quantity that is not stored as bf16 is
 * held in `hgdo_real`, which is double in the default build (libhgd_oracle.so)
 * and float in the second build (libhgd_oracle_f32.so, the "fp32 reference"
 * the pages compare against).  hgdo_real_bytes() tells the caller which.
 * Rounding to bf16 happens only at the rounding points listed for each routine
 * (round-to-nearest-even, computed directly from the exact value).
 *
 * Sources (page title -- section):
 *   [TF]   "qwen3_5 cuda: mixed-width MLX checkpoints ... #849" -- PR body: gated delta
 *          rule, causal convolution and gated attention at bf16 rounding points;
 *          windows of up to 16 rows equal one-row steps bit for bit; attention in
 *          key chunks cut at logical positions.
 *   [LUCE] "luce-megakernel HANDOFF.md" -- Model: 24 layers, [DN,DN,DN,FA] x 6.
 *   [FT]   "Running on Turing (sm_75)" -- What was checked: RMSNorm, causal conv,
 *          GDN decode, gated RMSNorm, silu_and_mul, the 248k-row lm_head; the
 *          GDN state is stored [num_heads, V, K].
 *   [AST]  "decode_linear_benchmark.md" -- commit message: BF16 GEMV, fused
 *          up/gate SwiGLU; error metrics: max abs, relative L2, row argmax.
 *   [MOE]  "nvfp4-megamoe-kernel commit log" -- stable softplus
 *          max(x,0)+log1p(exp(-|x|)); top-k ties go to the lower index.
 *   The recurrence, S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,
 *   o_t = S_t q_t with L2-normalised q,k, a = exp(g), b = sigmoid(b_raw), is the
 *   gated delta rule in its standard published form; the pages ([TF], [LUCE]
 *   Model) name it without writing it out.
 */
#ifndef HGD_ORACLE_H
#define HGD_ORACLE_H

#include <stdint.h>

#ifndef HGDO_REAL
#define HGDO_REAL double
#endif
typedef HGDO_REAL hgdo_real;

#ifdef __cplusplus
extern "C" {
#endif

/* sizeof(hgdo_real): 8 for the default build, 4 for the fp32 build. */
int hgdo_real_bytes(void);

/* bf16 <-> real.  bf16 values are 16-bit patterns (the upper half of an IEEE
 * binary32).  hgdo_round_bf16 rounds the exact real value to the nearest bf16,
 * ties to even, with overflow to +-inf and NaN kept as a quiet NaN. */
hgdo_real hgdo_bf16_value(uint16_t h);
uint16_t hgdo_round_bf16(hgdo_real v);
void hgdo_round_bf16_array(const hgdo_real* v, uint16_t* out, int64_t n);

/* y[m][n] = sum_k x[m][k] * W[n][k]   ([AST] BF16 GEMV; W is [N,K] row-major,
 * x is [M,K], y is [M,N] in hgdo_real, no rounding). */
void hgdo_gemv(const uint16_t* W, const uint16_t* x, hgdo_real* y, int M, int N, int K);

/* h[m][i] = bf16( silu(g) * u ),  g = sum_k x[m][k] Wg[i][k],  u = sum_k x[m][k] Wu[i][k]
 * ([AST] fused up/gate SwiGLU; [FT] silu_and_mul).  silu(t) = t / (1 + exp(-t)). */
void hgdo_swiglu(const uint16_t* Wg, const uint16_t* Wu, const uint16_t* x, uint16_t* h,
                 int M, int I, int K);

/* Depthwise causal conv1d over a kept tail ([TF] causal convolution, each row's
 * tail recorded).  Per stream b and channel c, for t = 0..T-1:
 *   s = sum_{j=0}^{kc-2} w[c][j] * tail[b][j][c]  +  w[c][kc-1] * x[b][t][c]
 *   y[b][t][c] = apply_silu ? silu(s) : s
 *   tail[b][j][c] <- tail[b][j+1][c] (j < kc-2),  tail[b][kc-2][c] <- x[b][t][c]
 * tail is oldest-first, [B][kc-1][C], updated in place.  If tail_rec is not
 * NULL it receives the tail after each row: [B][T][kc-1][C]. */
void hgdo_conv1d_tail_update(const hgdo_real* x, hgdo_real* tail, const uint16_t* w,
                             hgdo_real* y, hgdo_real* tail_rec,
                             int B, int T, int C, int kc, int apply_silu);

/* Gated delta rule, dense form, one row at a time.
 * Row (b,t), head h:  q = q_ptr + (b*T+t)*row_stride + h*dk  (k likewise),
 *                     v = v_ptr + (b*T+t)*row_stride + h*dv,
 *                     g = g[(b*T+t)*H + h],  braw likewise.
 *   if l2norm: q <- q / sqrt(sum q^2 + 1e-6), k likewise
 *   alpha = exp(g),  beta = 1 / (1 + exp(-braw))
 *   A = I - beta k k^T                                (dk x dk, formed explicitly)
 *   S <- alpha (S A) + beta v k^T                     (S is [dv][dk])
 *   o = S q                                           (the UPDATED state)
 * S is [B][H][dv][dk] ([FT]: state stored [num_heads, V, K]), updated in place.
 * o is [B][T][H][dv].  S_rec, if not NULL, gets S after each row:
 * [B][T][H][dv][dk]. */
void hgdo_gdn_step(const hgdo_real* q, const hgdo_real* k, const hgdo_real* v, int64_t row_stride,
                   const hgdo_real* g, const hgdo_real* braw, hgdo_real* S, hgdo_real* o,
                   hgdo_real* S_rec, int B, int T, int H, int dk, int dv, int l2norm);

/* The same with H value heads over Hk query/key heads (H a multiple of Hk;
 * [TF] commit on config.json widths: linear value heads over fewer key heads):
 * value head h reads q and k of head h / (H / Hk) at q_ptr + row*row_stride +
 * (h / (H/Hk))*dk; v, g, braw, S, o and S_rec are per value head as above. */
void hgdo_gdn_step_grouped(const hgdo_real* q, const hgdo_real* k, const hgdo_real* v,
                           int64_t row_stride, const hgdo_real* g, const hgdo_real* braw,
                           hgdo_real* S, hgdo_real* o, hgdo_real* S_rec, int B, int T, int Hk,
                           int H, int dk, int dv, int l2norm);

/* Recurrence logs of a verify window ([TF] tree-window commit note: each stream
 * logs its rows' decay, write and key; keep replays the kept rows onto the
 * recurrence in one pass).  Same inputs and outputs o as hgdo_gdn_step, but S
 * is left as it is; the rows run on a copy, and for row (b,t), head h:
 *   log_alpha[b][t][h]    = alpha = exp(g)
 *   log_k[b][t][h][dk]    = k (L2-normalised when l2norm, as the step uses it)
 *   log_delta[b][t][h][dv] = beta (v - alpha S_{t-1} k)    (S_{t-1}: state before the row)
 * so that S_t = alpha S_{t-1} + delta k^T. */
void hgdo_gdn_window_log(const hgdo_real* q, const hgdo_real* k, const hgdo_real* v, int64_t row_stride,
                         const hgdo_real* g, const hgdo_real* braw, const hgdo_real* S, hgdo_real* o,
                         hgdo_real* log_alpha, hgdo_real* log_delta, hgdo_real* log_k,
                         int B, int T, int H, int dk, int dv, int l2norm);

/* keep: for each stream b, S[b] <- alpha_t S[b] + delta_t k_t^T for t = 0 ..
 * keep[b]-1 from the logs above (T rows per stream).  Returns 2 (nothing
 * changed) if some keep[b] is outside [0, T]. */
int hgdo_gdn_keep(hgdo_real* S, const hgdo_real* log_alpha, const hgdo_real* log_delta,
                  const hgdo_real* log_k, const int32_t* keep, int B, int T, int H, int dk, int dv);

/* The conv tail [B][kc-1][C] after the first keep[b] rows of a window with inputs
 * x [B][T][C]: each kept row shifts the tail by one and becomes its newest entry.
 * Returns 2 (nothing changed) if some keep[b] is outside [0, T]. */
int hgdo_conv1d_keep(hgdo_real* tail, const hgdo_real* x, const int32_t* keep, int B, int T, int C, int kc);

/* softplus(t) = max(t,0) + log1p(exp(-|t|))  ([MOE] activation_topk's stable form). */
hgdo_real hgdo_softplus(hgdo_real t);

/* Log-decay of the stack's GDN layers, per head h < H:
 *   g[h] = -exp(A_log[h]) * softplus(a[h] + dt_bias[h])
 * a[h] is the head's "a" projection output (real); A_log and dt_bias are the
 * layer's bf16 parameters.  The state update then uses alpha = exp(g). */
void hgdo_gdn_gates(const hgdo_real* a, const uint16_t* A_log, const uint16_t* dt_bias,
                    hgdo_real* g, int H);

/* y[m] = bf16( x[m] * (1/sqrt(mean(x[m]^2) + eps)) * w )   ([FT] RMSNorm). */
void hgdo_rmsnorm(const uint16_t* x, const uint16_t* w, uint16_t* y, int M, int D, double eps);

/* Per head of width d: u = bf16( o * (1/sqrt(mean(o^2)+eps)) * w * silu(z) )
 * ([FT] gated RMSNorm).  o is real, z and w are bf16; o,z,u are [M][nh*d]. */
void hgdo_gated_rmsnorm(const hgdo_real* o, const uint16_t* z, const uint16_t* w, uint16_t* u,
                        int M, int nh, int d, double eps);

/* Rotate-half rotary embedding of one head vector x[hd] at absolute position
 * pos, base `base`:  for i < hd/2, th = pos * base^(-2i/hd),
 *   x'[i] = x[i] cos th - x[i+hd/2] sin th,  x'[i+hd/2] = x[i+hd/2] cos th + x[i] sin th. */
void hgdo_rope(hgdo_real* x, int hd, int pos, double base);

/* Decode attention for one query row ([TF] gated attention; GQA: query head i
 * reads key/value head i / (nq/nkv)).  Kc, Vc are the stream's caches
 * [nkv][Lmax][hd] bf16; keys 0..nkeys-1 are attended.  q is the already
 * rotated [nq][hd]; gate is [nq][hd].  out[i] = bf16( softmax(q_i K^T / sqrt(hd)) V
 * * sigmoid(gate_i) ), [nq][hd]. */
void hgdo_attention_row(const hgdo_real* q, const hgdo_real* gate, const uint16_t* Kc,
                        const uint16_t* Vc, int nkeys, int Lmax, int nq, int nkv, int hd,
                        uint16_t* out);

/* ---------------------------------------------------------------- stack --- */

typedef struct hgdo_config {
    int32_t n_layers;       /* 24 */
    int32_t hidden;         /* D */
    int32_t vocab;          /* V */
    int32_t gdn_heads;      /* Hk: GDN query/key heads */
    int32_t gdn_dk;
    int32_t gdn_dv;
    int32_t conv_k;         /* kc */
    int32_t attn_q_heads;   /* nq */
    int32_t attn_kv_heads;  /* nkv */
    int32_t attn_head_dim;  /* hd */
    int32_t mlp_inter;      /* I */
    int32_t attn_every;     /* layer l is attention iff l % attn_every == attn_every-1 */
    double norm_eps;
    double rope_base;
    int32_t gdn_v_heads;    /* value heads Hv (a multiple of gdn_heads); 0 = gdn_heads */
} hgdo_config;

/* One layer's weights, all bf16, row-major [out, in] (Hk key heads, H value heads):
 *  GDN layer: in_norm[D]; w_in [2*Hk*dk + 2*H*dv + 2*H, D] with output rows
 *    q (Hk*dk) | k (Hk*dk) | v (H*dv) | z (H*dv) | a (H) | b (H);
 *    conv_w [2*Hk*dk + H*dv, kc] over the channels q|k|v; A_log[H]; dt_bias[H];
 *    gnorm_w[dv]; w_out [D, H*dv].
 *  Attention layer: in_norm[D]; w_in [2*nq*hd + 2*nkv*hd, D] with output rows
 *    q (nq*hd) | gate (nq*hd) | k (nkv*hd) | v (nkv*hd); w_out [D, nq*hd].
 *  Both: post_norm[D]; w_gate, w_up [I, D]; w_down [D, I]. */
typedef struct hgdo_layer {
    const uint16_t* in_norm;
    const uint16_t* w_in;
    const uint16_t* conv_w;
    const uint16_t* A_log;
    const uint16_t* dt_bias;
    const uint16_t* gnorm_w;
    const uint16_t* w_out;
    const uint16_t* post_norm;
    const uint16_t* w_gate;
    const uint16_t* w_up;
    const uint16_t* w_down;
} hgdo_layer;

#define HGDO_MAX_LAYERS 64

typedef struct hgdo_model {
    hgdo_config cfg;
    const uint16_t* embed;      /* [V, D] */
    const uint16_t* final_norm; /* [D] */
    hgdo_layer layers[HGDO_MAX_LAYERS];
    const uint16_t* lm_head;    /* [V, D], or NULL: the head is tied to the embedding */
} hgdo_model;

/* Per-stream decode state.  n_gdn / n_attn are the numbers of GDN / attention
 * layers in layer order.
 *   S    [n_gdn][B][H][dv][dk]        real (H value heads)
 *   tail [n_gdn][B][kc-1][C]          real, C = 2*Hk*dk + H*dv
 *   kv   [n_attn][2][B][nkv][Lmax][hd] bf16 (index 0 = keys, already rotated)
 *   pos  [B]  absolute position of the next row of each stream */
typedef struct hgdo_state {
    hgdo_real* S;
    hgdo_real* tail;
    uint16_t* kv;
    int32_t* pos;
    int32_t B;
    int32_t Lmax;
} hgdo_state;

/* One decode call: T rows for each of B streams, tokens[b*T + t].
 * Row (b,t) sits at position pos[b]+t and attends its stream's keys 0..pos[b]+t.
 * Rows are processed one at a time, stream by stream, through all layers:
 *   x = E[token]                                            (bf16 residual stream)
 *   per layer:  h = bf16(RMSNorm(x) * in_norm)
 *     GDN:  p = W_in h;  conv(q|k|v) with SiLU;  z = bf16(p_z)
 *           g = hgdo_gdn_gates(a, A_log, dt_bias),  beta from b
 *           gated delta rule per value head (dense form; value head h reads
 *           key head h / (H/Hk));  u = bf16(gatedRMSNorm(o, z)) per value head
 *           x = bf16(x + W_out u)
 *     attn: p = W_in h;  RoPE(q), RoPE(k) at the row's position;
 *           K,V cache[pos] = bf16(k), bf16(v);  softmax attention over keys 0..pos
 *           times sigmoid(gate) -> bf16;  x = bf16(x + W_out attn)
 *     m = bf16(silu(W_gate hm) * (W_up hm)),  hm = bf16(RMSNorm(x) * post_norm)
 *     x = bf16(x + W_down m)
 *   logits = W_head * bf16(RMSNorm(x) * final_norm)   (real; W_head = lm_head, or the
 *            embedding E when lm_head is NULL: the tied head)
 *   argmax over the logits rounded to binary32, lowest index on ties ([MOE]).
 * logits [B*T][V] may be NULL.  argmax [B*T].  S_rec [n_gdn][B][T][H][dv][dk] and
 * tail_rec [n_gdn][B][T][kc-1][C] may be NULL.  x_rec [L][B][T][D] (bf16) may be
 * NULL: the residual stream after each layer.  pos[b] += T at the end.
 * Returns 0, or 1 if a logit was NaN (argmax then -1 for that row), 2 on bad
 * arguments (a position past Lmax, a token out of range, too many layers). */
int hgdo_decode_stack(const hgdo_model* m, hgdo_state* st, const int32_t* tokens, int T,
                      hgdo_real* logits, int32_t* argmax, hgdo_real* S_rec, hgdo_real* tail_rec,
                      uint16_t* x_rec);

#ifdef __cplusplus
}
#endif
#endif /* HGD_ORACLE_H */
