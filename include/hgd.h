/*
 * hgd.h -- C ABI of the B200 (sm_100a) hybrid gated-delta decode library.
 *
 * The library computes the small-batch decode step of a hybrid layer stack in
 * which three gated-delta-rule (GDN, "DeltaNet") layers alternate with one gated
 * full-attention layer, as the pages below describe it:
 *   [LUCE] "luce-megakernel HANDOFF.md" -- Model: 24 layers, [DN,DN,DN,FA] x 6;
 *          Architecture: one persistent decode kernel streaming all layers.
 *   [TF]   "qwen3_5 cuda: mixed-width MLX checkpoints ... #849" -- PR body: gated
 *          delta rule, causal convolution and gated attention at bf16 rounding
 *          points; windows of up to 16 rows that record each row's recurrence
 *          and convolution tail and equal one-row steps bit for bit; attention
 *          partials over key chunks cut at logical positions, then a merge.
 *   [FT]   "Running on Turing (sm_75)" -- What was checked: RMSNorm, causal conv,
 *          GDN decode, gated RMSNorm, silu_and_mul, the 248k-row lm_head; the GDN
 *          state is stored [num_heads, V, K]; debugging notes: an unchecked launch
 *          left outputs uninitialised.
 *   [AST]  "decode_linear_benchmark.md" -- commit message: BF16 GEMV and the fused
 *          up/gate SwiGLU primitive for decode shapes, M = 1..32.
 * The recurrence is the gated delta rule in its standard form (the pages name it
 * without writing it out):
 *   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t,
 *   q, k L2-normalised, alpha = exp(g), beta = sigmoid(b).
 *
 * Conventions for every entry point:
 *  - Every call returns an int status (HGD_OK = 0).  Nothing aborts or traps.  A
 *    rejected call launches nothing and writes nothing.
 *  - The caller owns every buffer.  The library allocates no device memory.
 *    Device pointers are plain CUDA device addresses of the current device;
 *    `stream` is a cudaStream_t (NULL = the legacy default stream).
 *  - Calls are asynchronous on `stream`; a launch failure is reported as
 *    HGD_ERR_CUDA (cudaGetLastError is consumed).  Errors found inside a kernel
 *    (a NaN logit, a wait that ran out) are written to a caller-provided device
 *    status word, read after the stream synchronises.
 *  - bf16 tensors are 16-bit bit patterns (uint16_t); row-major, contiguous.
 *    Weights use the [out, in] (Linear) layout.
 *  - Device pointers must be 16-byte aligned (HGD_ERR_MISALIGNED otherwise).
 *  - Only sm_100 devices are supported (HGD_ERR_UNSUPPORTED_DEVICE otherwise).
 */
#ifndef HGD_H
#define HGD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HGD_API __attribute__((visibility("default")))
#else
#define HGD_API
#endif

typedef struct CUstream_st* hgd_stream_t; /* same type as cudaStream_t */

enum hgd_status {
    HGD_OK = 0,
    HGD_ERR_INVALID_ARG = 1,        /* NULL where a buffer is required, negative size */
    HGD_ERR_UNSUPPORTED_SHAPE = 2,  /* a size outside what the kernels implement */
    HGD_ERR_MISALIGNED = 3,         /* a pointer that is not 16-byte aligned */
    HGD_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    HGD_ERR_TIMEOUT = 5,            /* a bounded in-kernel wait ran out (device status) */
    HGD_ERR_NOT_CORESIDENT = 6,     /* a persistent launch cannot keep all CTAs resident */
    HGD_ERR_NAN = 7,                /* a NaN logit reached the argmax (device status) */
    HGD_ERR_UNSUPPORTED_DEVICE = 8, /* the current device is not sm_100 */
    HGD_ERR_BUFFER_TOO_SMALL = 9    /* an arena smaller than the reported size */
};

/* Static text for a status code ("unknown status" for anything else). */
HGD_API const char* hgd_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
HGD_API int hgd_version(void);

/* ------------------------------------------------------------------ GEMV ---
 * y[m][n] = sum_k x[m][k] * W[n][k]   ([AST] BF16 GEMV for decode shapes).
 *   W  [N, K] bf16 device, x [M, K] bf16 device.
 *   y  [M, N] device: fp32 if y_is_fp32, else bf16 (round to nearest even).
 * fp32 accumulation.  Each output's arithmetic depends on K only, never on M,
 * N, the workspace or the device's SM count: a row computed in an M-row call
 * equals the same row computed alone, bit for bit.
 * workspace: optional device scratch of hgd_gemv_workspace_bytes(M, N, K, 0)
 * bytes that lets a GEMV with few output rows spread the K dimension over all
 * SMs (partials added in a fixed order).  NULL, or fewer bytes, runs without it
 * (same results, fewer SMs busy for small N).  It must be zero-filled before
 * its first use; every call leaves the counters in it back at zero, so it can be
 * reused without clearing.  Calls that share one workspace must not overlap on
 * the device.
 * Shapes: 1 <= M, 1 <= N, 32 <= K <= 65536 with K % 32 == 0
 * (HGD_ERR_UNSUPPORTED_SHAPE otherwise).  y must not overlap W, x or the
 * workspace. */
HGD_API int hgd_gemv_bf16(const uint16_t* W, const uint16_t* x, void* y, int y_is_fp32,
                  int M, int N, int K, void* workspace, size_t workspace_bytes,
                  hgd_stream_t stream);

/* Bytes of the optional split-K workspace of a GEMV (swiglu = 0) or a fused
 * SwiGLU (swiglu = 1, N = I) of this shape; 0 when that shape never uses one. */
HGD_API int hgd_gemv_workspace_bytes(int M, int N, int K, int swiglu, size_t* bytes);

/* ------------------------------------------------------------ diagnostics ---
 * Check that a stuck in-kernel wait ends with a status rather than a hang (the
 * conventions above: errors found inside a kernel go to a device status word):
 * one kernel runs the bounded mbarrier wait the weight rings and the tensor-core
 * GEMM use, on a barrier that nothing completes.  About 2 s later the wait runs
 * out and the kernel writes HGD_ERR_TIMEOUT to *status (device int32, 16-byte
 * aligned; not cleared first).  Launches nothing else; the context stays usable. */
HGD_API int hgd_check_bounded_wait(int32_t* status, hgd_stream_t stream);

/* ------------------------------------------------------- tensor-core GEMM ---
 * The same product for windows of many token rows ([TF] PR body: windows of up
 * to 16 rows per stream, several streams per call; [AST] commit message: the
 * decode projections as GEMVs): at 16..256 rows the projection is a dense
 * contraction and runs on the 5th-generation tensor cores (tcgen05.mma, fp32
 * accumulators in tensor memory).
 *   y[m][n] = sum_k x[m][k] * W[n][k],  fp32 out [M, N] (row-major).
 * The weight is packed once (hgd_gemm_tc_pack_weight) into 128 x 64 tiles in the
 * tensor core's core-matrix order; the call packs x into its workspace, streams
 * each tile once, and splits K over at most 8 CTAs by a fixed function of N
 * and K (the splits of a 128-row block run as one thread-block cluster and add
 * their partials in split order through shared memory), so results do not
 * depend on the device or the call's neighbours.  The sums follow the tensor core's order, not the
 * GEMV's: results agree with hgd_gemv_bf16 to fp32 rounding, not bit for bit.
 * Shapes: 1 <= M <= 256, 1 <= N, 64 <= K <= 65536 with K % 64 == 0
 * (HGD_ERR_UNSUPPORTED_SHAPE otherwise). */
/* Bytes of the packed weight of an [N, K] matrix (N rounded up to 128 rows). */
HGD_API int hgd_gemm_tc_weight_bytes(int N, int K, size_t* bytes);
/* W [N, K] bf16 (device) -> Wp (device, hgd_gemm_tc_weight_bytes bytes; the
 * rows past N are zero).  Wp must be complete before a GEMM reads it: the GEMM
 * starts streaming it before it waits for the kernel that precedes it on the
 * stream, so that kernel must not be the one writing Wp. */
HGD_API int hgd_gemm_tc_pack_weight(const uint16_t* W, uint16_t* Wp, int N, int K, hgd_stream_t stream);
/* Bytes of the workspace of a GEMM of this shape (the packed token rows). */
HGD_API int hgd_gemm_tc_workspace_bytes(int M, int N, int K, size_t* bytes);
/* The plan of a GEMM of this shape, for inspection: *splits, the CTAs (one
 * cluster) that share each 128-row block's K range (a power of two, 1..8, a
 * function of N and K only), and *stages, its shared-memory pipeline depth.
 * Same shape rules as hgd_gemm_tc_bf16; no device work. */
HGD_API int hgd_gemm_tc_plan(int M, int N, int K, int* splits, int* stages);
/* Wp: packed weight; x [M, K] bf16; y [M, N] fp32; workspace of at least
 * hgd_gemm_tc_workspace_bytes bytes (HGD_ERR_BUFFER_TOO_SMALL otherwise; no
 * initial contents needed; calls sharing one must not overlap on the device);
 * status: optional device int32, set to HGD_ERR_TIMEOUT if an in-kernel wait ran
 * out (y is then not written).  y must not overlap the other buffers. */
HGD_API int hgd_gemm_tc_bf16(const uint16_t* Wp, const uint16_t* x, float* y, int M, int N, int K,
                     void* workspace, size_t workspace_bytes, int32_t* status, hgd_stream_t stream);

/* hgd_gemv_bf16 for callers that cannot allocate device memory (a plugin whose
 * host framework owns the device allocator and offers it no handle; a decode
 * loop that must never wait on the synchronisation a cudaMalloc brings).  The
 * pages have no counterpart: it exists only so such callers need no workspace.
 * Same inputs, output, shapes and results as hgd_gemv_bf16, but the split-K
 * scratch is a 4 MiB array built into the library, present on every device that
 * loads it until the process exits.  Nothing is allocated.
 *  - The first call in a CUDA context looks the array's device address up (once
 *    per context, with that context current: once per device in the usual
 *    runtime use, and again after a device reset, which starts a new context);
 *    make that first call before capturing any stream into a CUDA graph.
 *    Concurrent first calls from several host threads are safe.
 *  - A shape whose scratch would exceed 4 MiB returns HGD_ERR_BUFFER_TOO_SMALL
 *    and launches nothing (hgd_gemv_workspace_bytes tells the size needed).
 *  - Each call clears the part of the array that must start at zero (its
 *    counters) on `stream` before the GEMV; the rest keeps the last call's data.
 *  - All calls share the one array: calls that overlap on the device (other
 *    streams, other host threads) race and corrupt each other's results.
 *    Issue them on one stream, or order them. */
HGD_API int hgd_gemv_bf16_static_ws(const uint16_t* W, const uint16_t* x, void* y, int y_is_fp32,
                                    int M, int N, int K, hgd_stream_t stream);

/* h[m][i] = bf16( silu(g) * u ),  g = x . W_gate[i],  u = x . W_up[i]
 * ([AST] fused BF16 up/gate SwiGLU; [FT] silu_and_mul), silu(t) = t/(1+exp(-t)).
 *   W_gate, W_up [I, K] bf16 device; x [M, K] bf16 device; h [M, I] bf16 device.
 * g and u are fp32 dot products computed exactly as hgd_gemv_bf16 computes them.
 * Shapes and workspace as hgd_gemv_bf16 with N = I (workspace size with swiglu = 1). */
HGD_API int hgd_gemv_swiglu_bf16(const uint16_t* W_gate, const uint16_t* W_up, const uint16_t* x,
                         uint16_t* h, int M, int I, int K, void* workspace,
                         size_t workspace_bytes, hgd_stream_t stream);

/* -------------------------------------------------------- conv1d tail ---
 * Depthwise causal conv1d over a kept tail ([TF] causal convolution with each
 * row's tail recorded).  For stream b, channel c and row t = 0..T-1:
 *   s = sum_{j<kc-1} w[c][j] * tail[b][j][c] + w[c][kc-1] * x[b][t][c]
 *   y[b][t][c] = apply_silu ? silu(s) : s
 *   tail[b][:, c] shifts by one row and takes x[b][t][c] as its newest entry.
 *   x [B, T, C] fp32, tail [B, kc-1, C] fp32 (oldest first, updated in place),
 *   w [C, kc] bf16, y [B, T, C] fp32, tail_rec [B, T, kc-1, C] fp32 or NULL
 *   (the tail after each row).  All device pointers.
 * Shapes: B, T, C >= 1; 2 <= kc <= 8.  A T-row call equals T one-row calls
 * bit for bit. */
HGD_API int hgd_conv1d_tail_update(const float* x, float* tail, const uint16_t* w, float* y,
                           float* tail_rec, int B, int T, int C, int kc, int apply_silu,
                           hgd_stream_t stream);

/* ---------------------------------------------------- gated delta rule ---
 * One or more recurrent rows of the gated delta rule per (stream, head), state
 * updated in place in fp32 ([FT] state layout [heads, V, K]).
 * Row (b,t), head h reads
 *   q = q_ptr + (b*T+t)*row_stride + h*dk,  k likewise,  v = v_ptr + (b*T+t)*row_stride + h*dv,
 *   g[(b*T+t)*H + h], b[(b*T+t)*H + h]   (raw: alpha = exp(g), beta = sigmoid(b)),
 * and computes, with q,k L2-normalised over dk (x / sqrt(sum x^2 + 1e-6)) when
 * l2norm_qk is set:
 *   S <- alpha S + beta (v - alpha S k) k^T     (= alpha S (I - beta k k^T) + beta v k^T)
 *   o = S q                                     (with the updated S)
 *   S [B, H, dv, dk] fp32 device, in place.
 *   o [B, T, H, dv] fp32 device; o_bf16 the same shape in bf16, or NULL.
 *   S_rec [B, T, H, dv, dk] fp32 device or NULL: S after each row.
 * row_stride (elements, >= H*dk and >= H*dv) lets q|k|v come packed in one
 * [B*T, row_stride] array (e.g. a conv output); for separate contiguous
 * [B,T,H,d] arrays pass H*dk.
 * Shapes: dk in {32, 64, 128, 256}; dv a multiple of 16 up to 1024; H, B, T >= 1.
 * A T-row call equals T one-row calls bit for bit. */
HGD_API int hgd_gdn_decode_step(const float* q, const float* k, const float* v, int64_t row_stride,
                        const float* g, const float* b, float* S, float* o, uint16_t* o_bf16,
                        float* S_rec, int B, int T, int H, int dk, int dv, int l2norm_qk,
                        hgd_stream_t stream);

/* The same rows with H value heads over Hk query/key heads ([TF] commit on the
 * widths read from config.json: linear value heads over fewer key heads; H a
 * multiple of Hk): value head h reads q and k of head h / (H / Hk), at
 * q_ptr + (b*T+t)*row_stride + (h / (H/Hk))*dk; v, g, b, S, o, o_bf16 and S_rec
 * are per value head exactly as above.  Hk = H is hgd_gdn_decode_step.
 * row_stride >= Hk*dk and >= H*dv. */
HGD_API int hgd_gdn_decode_step_grouped(const float* q, const float* k, const float* v,
                                        int64_t row_stride, const float* g, const float* b, float* S,
                                        float* o, uint16_t* o_bf16, float* S_rec, int B, int T, int Hk,
                                        int H, int dk, int dv, int l2norm_qk, hgd_stream_t stream);

/* -------------------------------------------------------------- prefill ---
 * The rows of a prompt ([LUCE] Architecture Summary: a prefill kernel beside the
 * decode kernel; Expected Results: pp512): the same state and outputs as
 * hgd_gdn_decode_step over the T rows (same q, k, v, row_stride, g, b, S, o and
 * layouts), computed a chunk of 32 rows at a time: within a chunk the rows'
 * writes solve the unit lower-triangular system (I + A) U = diag(beta) (V -
 * diag(Gamma) K S_0^T) with A[t][s] = beta_t (Gamma_t / Gamma_s) (k_s . k_t),
 * Gamma the running product of alpha, and the outputs and the next state follow
 * from U in matrix products.  fp32 throughout; equal to the one-row steps to
 * fp32 rounding (not bit for bit).  No per-row state records.
 * Shapes: dk in {64, 128}; dv a multiple of 32 up to 1024; row_stride a
 * multiple of 4 (q, k rows 16-byte aligned). */
HGD_API int hgd_gdn_prefill(const float* q, const float* k, const float* v, int64_t row_stride,
                            const float* g, const float* b, float* S, float* o, int B, int T, int H,
                            int dk, int dv, int l2norm_qk, hgd_stream_t stream);

/* ------------------------------------------ recurrence logs and keep ---
 * [TF] tree-window commit note: a verify window no longer snapshots every row's
 * state; each stream logs its rows' decay, write and key, and keep replays the
 * kept rows onto the recurrence in one pass.  Row t of a head updates
 *   S_t = alpha_t S_{t-1} + delta_t k_t^T,   delta_t = beta_t (v_t - alpha_t S_{t-1} k_t)
 * (the gated delta rule above, rewritten), so (alpha_t, delta_t, k_t) carry the
 * row: 4 * (1 + dv + dk) bytes a head instead of the 4 * dv * dk of a snapshot.
 *
 * hgd_gdn_window_log: the rows of hgd_gdn_decode_step (same q, k, v, g, b,
 * row_stride, o, o_bf16, shapes), but S is only read: every row runs on the
 * state as the rows before it left it, and nothing is written back.  Per row
 * (b,t) and head h it writes
 *   log_alpha [B,T,H]     alpha = exp(g)
 *   log_delta [B,T,H,dv]  the write delta
 *   log_k     [B,T,H,dk]  k as the row used it (L2-normalised if l2norm_qk)
 * (fp32 device arrays).  o equals the o of hgd_gdn_decode_step bit for bit. */
HGD_API int hgd_gdn_window_log(const float* q, const float* k, const float* v, int64_t row_stride,
                               const float* g, const float* b, const float* S, float* o,
                               uint16_t* o_bf16, float* log_alpha, float* log_delta, float* log_k,
                               int B, int T, int H, int dk, int dv, int l2norm_qk,
                               hgd_stream_t stream);

/* keep: S [B,H,dv,dk] (fp32 device, in place) takes the first keep[b] logged
 * rows of stream b, S <- alpha_t S + delta_t k_t^T for t = 0..keep[b]-1, with
 * the logs of a T-row hgd_gdn_window_log call.  keep [B] int32 is read on the
 * device (so an accept decision made by a kernel needs no host round trip).
 * S after keep(n) equals S after n one-row hgd_gdn_decode_step calls bit for
 * bit.  A keep[b] outside [0, T] leaves stream b as it is and writes
 * HGD_ERR_INVALID_ARG to *status_dev (device int32, or NULL). */
HGD_API int hgd_gdn_keep(float* S, const float* log_alpha, const float* log_delta, const float* log_k,
                         const int32_t* keep, int32_t* status_dev, int B, int T, int H, int dk, int dv,
                         hgd_stream_t stream);

/* The conv tail's keep: tail [B, kc-1, C] (fp32 device, in place) takes the
 * first keep[b] rows of the window's conv inputs x [B, T, C] (each row shifts
 * the tail by one and becomes its newest entry), which equals the tail
 * hgd_conv1d_tail_update leaves after those rows, bit for bit.  keep and
 * status_dev as hgd_gdn_keep.  Shapes: 2 <= kc <= 8. */
HGD_API int hgd_conv1d_keep(float* tail, const float* x, const int32_t* keep, int32_t* status_dev,
                            int B, int T, int C, int kc, hgd_stream_t stream);

/* ------------------------------------------------------ decode stack ---- */

/* Geometry of the hybrid stack ([LUCE] Model).  Layer l is a gated-attention
 * layer iff l % attn_every == attn_every - 1, otherwise a GDN layer. */
typedef struct hgd_config {
    int32_t n_layers;      /* 24 */
    int32_t hidden;        /* D = 1024 */
    int32_t vocab;         /* 248320; the LM head is tied to the embedding */
    int32_t gdn_heads;     /* H = 16 */
    int32_t gdn_dk;        /* 128 */
    int32_t gdn_dv;        /* 128 */
    int32_t conv_k;        /* 4 */
    int32_t attn_q_heads;  /* 8 */
    int32_t attn_kv_heads; /* 2 */
    int32_t attn_head_dim; /* 256 */
    int32_t mlp_inter;     /* I = 3584 */
    int32_t attn_every;    /* 4 */
    float norm_eps;        /* 1e-6 */
    float rope_base;       /* 10000 */
    /* [TF] commit on the widths read from config.json: linear value heads over
     * fewer key heads, an untied head. */
    int32_t gdn_v_heads;   /* GDN value heads Hv, a multiple of gdn_heads (the
                              query/key heads); 0 = gdn_heads.  Value head h reads
                              query/key head h / (Hv / gdn_heads). */
    int32_t untied_head;   /* 0: the LM head is the embedding; 1: its own [V, D]
                              tensor HGD_W_LM_HEAD */
} hgd_config;

#define HGD_MAX_LAYERS 64

/* Tensors of the weight arena.  Per layer (layer >= 0):                 */
enum hgd_weight_tensor {
    HGD_W_IN_NORM = 0,   /* [D] gain (bf16) */
    /* (GDN: Hk = gdn_heads query/key heads, H = value heads, see hgd_config) */
    HGD_W_IN = 1,        /* GDN: [2*Hk*dk + 2*H*dv + 2*H, D], rows q|k|v|z|a|b
                            attention: [2*nq*hd + 2*nkv*hd, D], rows q|gate|k|v */
    HGD_W_CONV = 2,      /* GDN: [2*Hk*dk + H*dv, kc] over channels q|k|v */
    HGD_W_A_LOG = 3,     /* GDN: [H] */
    HGD_W_DT_BIAS = 4,   /* GDN: [H] */
    HGD_W_GNORM = 5,     /* GDN: [dv] gated-RMSNorm gain shared by heads */
    HGD_W_OUT = 6,       /* GDN: [D, H*dv]; attention: [D, nq*hd] */
    HGD_W_POST_NORM = 7, /* [D] */
    HGD_W_GATE = 8,      /* [I, D] */
    HGD_W_UP = 9,        /* [I, D] */
    HGD_W_DOWN = 10,     /* [D, I] */
    HGD_W_LAYER_COUNT = 11,
    /* model-level tensors (layer = -1) */
    HGD_W_EMBED = 100,      /* [V, D], also the LM head unless untied_head */
    HGD_W_FINAL_NORM = 101, /* [D] */
    HGD_W_LM_HEAD = 102     /* [V, D], present only with untied_head */
};

/* Model handle.  Filled by hgd_model_init from a caller-owned weight arena;
 * holds only pointers into it and the configuration. */
typedef struct hgd_model {
    hgd_config cfg;
    const uint16_t* embed;
    const uint16_t* final_norm;
    const uint16_t* w[HGD_MAX_LAYERS][HGD_W_LAYER_COUNT];
    size_t arena_bytes;
    const uint16_t* lm_head;  /* HGD_W_LM_HEAD with untied_head, else NULL (the embedding serves) */
    /* the tensor-core chain's weights (hgd_model_attach_tc), else NULL: per layer
     * in-projection, out-projection, gate+up, down; the head */
    const uint16_t* tcw[HGD_MAX_LAYERS][4];
    const uint16_t* tc_head;
} hgd_model;

/* Bytes of the weight arena for `cfg` (every tensor 256-byte aligned). */
HGD_API int hgd_model_arena_bytes(const hgd_config* cfg, size_t* bytes);

/* Byte offset and logical element count of one tensor in the weight arena.  A
 * tensor the layer does not have (e.g. HGD_W_CONV in an attention layer)
 * reports numel = 0.  HGD_ERR_INVALID_ARG for an unknown tensor or layer.
 * The projection matrices (HGD_W_IN, HGD_W_OUT, HGD_W_GATE + HGD_W_UP, which
 * share one region, HGD_W_DOWN and HGD_W_EMBED) are stored in the GEMV engine's
 * fragment order, not row-major: fill the arena with hgd_model_load_tensor. */
HGD_API int hgd_model_tensor(const hgd_config* cfg, int layer, int tensor, size_t* offset,
                     size_t* numel);

/* Store one tensor into the weight arena from a row-major bf16 copy `src`
 * (device, [out, in] for matrices, numel as hgd_model_tensor reports), packing
 * the projection matrices into the fragment order the kernels stream.  `arena`
 * is the device arena of hgd_model_arena_bytes bytes (256-byte aligned).
 * Asynchronous on `stream`; `src` must stay valid until the stream reaches the
 * call.  Returns HGD_ERR_INVALID_ARG for a tensor the layer does not have. */
HGD_API int hgd_model_load_tensor(const hgd_config* cfg, void* arena, size_t arena_bytes, int layer,
                                  int tensor, const uint16_t* src, hgd_stream_t stream);

/* Validate cfg and point `m` at the arena (device memory filled through
 * hgd_model_load_tensor).  No allocation, no launch. */
HGD_API int hgd_model_init(hgd_model* m, const hgd_config* cfg, const void* weight_arena, size_t bytes);

/* Tensors of the state arena (per-stream recurrent state, KV cache, position,
 * and the activation scratch of one call). */
enum hgd_state_tensor {
    HGD_S_GDN = 0,    /* [n_gdn, B, H, dv, dk] fp32 recurrent state (H value heads) */
    HGD_S_CONV = 1,   /* [n_gdn, B, kc-1, 2*Hk*dk + H*dv] fp32 conv tails, oldest first */
    HGD_S_KV = 2,     /* [n_attn, 2, B, nkv, Lmax, hd] bf16 (0 = keys, rotated) */
    HGD_S_POS = 3,    /* [B] int32 position of each stream's next row */
    HGD_S_RESID = 4,  /* [B*Tmax, D] bf16 residual stream of the current call */
    HGD_S_COUNT = 5
};

typedef struct hgd_state {
    int32_t B, Tmax, Lmax;
    void* arena;
    size_t arena_bytes;
    size_t off[32];  /* byte offsets of the state tensors and scratch buffers */
} hgd_state;

/* Bytes of the state arena for B streams, up to Tmax rows per call and Lmax
 * cache positions.  Shapes: B*Tmax <= 256, Lmax <= 16384. */
HGD_API int hgd_state_arena_bytes(const hgd_config* cfg, int B, int Tmax, int Lmax, size_t* bytes);

/* Byte offset and element count of a caller-visible state tensor. */
HGD_API int hgd_state_tensor(const hgd_config* cfg, int B, int Tmax, int Lmax, int tensor,
                     size_t* offset, size_t* numel);

/* Lay the state out in `state_arena` (caller-owned device memory of at least
 * hgd_state_arena_bytes, zero-filled before its first use: it also holds the
 * split-K workspace, whose counters every call leaves at zero).  The caller
 * initialises S, conv tails, KV rows below each stream's position and the
 * positions themselves; nothing is written here. */
HGD_API int hgd_state_init(hgd_state* st, const hgd_model* m, int B, int Tmax, int Lmax,
                   void* state_arena, size_t bytes);

/* One decode call over T rows of each of B streams ([LUCE] decode step;
 * [TF] windows of rows that equal one-row steps):
 *   tokens [B, T] int32 device; row (b,t) sits at position pos[b]+t and attends
 *   its stream's keys 0..pos[b]+t.
 *   logits [B*T, V] fp32 device or NULL; argmax [B*T] int32 device (first
 *   maximum, lowest index on ties).
 *   S_rec [n_gdn, B, T, H, dv, dk] and tail_rec [n_gdn, B, T, kc-1, C] fp32
 *   device or NULL: the recurrent state and conv tail after each row.
 *   status_dev: int32 device word; the kernels write a nonzero hgd_status there
 *   on an in-kernel error (it is not cleared; zero it before the call).
 * Every step is on `stream` and reads sizes from the device, so a call can be
 * captured in a CUDA graph and replayed while positions advance.  pos[b] += T
 * at the end.  Requires 1 <= T <= Tmax and pos[b]+T <= Lmax (checked on the
 * device: violation sets HGD_ERR_INVALID_ARG in status_dev and skips the row). */
HGD_API int hgd_decode_layer_stack(const hgd_model* m, const hgd_state* st, const int32_t* tokens,
                           int T, float* logits, int32_t* argmax, float* S_rec,
                           float* tail_rec, int32_t* status_dev, hgd_stream_t stream);

/* Part of one decode call: layers [layer_begin, layer_end) and, if run_head, the
 * final RMSNorm, the tied LM head, the argmax and the position advance.
 * The residual stream of the call's B*T rows lives in the state tensor
 * HGD_S_RESID ([B*Tmax, D] bf16, rows b*T + t): a range that starts at layer 0
 * gathers the embedding rows of `tokens` into it; a range that starts later
 * reads it as left by the previous range (or as written by the caller), and
 * every range leaves it holding the output of its last layer.  Running
 * [0, a), [a, b), ..., [c, L) + head on one stream equals one
 * hgd_decode_layer_stack call bit for bit.  tokens may be NULL when
 * layer_begin > 0; argmax may be NULL when run_head is 0.  Positions advance
 * only with the head, so ranges of one call all see the call's positions. */
HGD_API int hgd_decode_layer_stack_range(const hgd_model* m, const hgd_state* st, const int32_t* tokens,
                                         int T, int layer_begin, int layer_end, int run_head,
                                         float* logits, int32_t* argmax, float* S_rec, float* tail_rec,
                                         int32_t* status_dev, hgd_stream_t stream);

/* ----------------------------------------------------- verify windows ---
 * [TF] tree-window commit note: a verify window no longer snapshots every row's
 * state; each stream logs its rows' decay, write and key, and keep replays the
 * kept rows onto the recurrence in one pass; one-row steps update in place.
 *
 * hgd_decode_layer_stack_verify: one decode call over T rows of each stream,
 * with the logits and argmax of hgd_decode_layer_stack (bit for bit: the same
 * kernels), that leaves the recurrent state as it found it:
 *  - the GDN layers log each row's (alpha, delta, k) instead of writing S;
 *  - the causal conv runs on a copy of the tails kept in the log and logs each
 *    row's conv input;
 *  - the attention layers write K/V at positions pos[b]..pos[b]+T-1 as usual
 *    (rows past what keep accepts are overwritten by later calls);
 *  - positions do not advance.
 * `log` is caller-owned device memory of hgd_verify_log_bytes(cfg, B, T) bytes,
 * 256-byte aligned (HGD_ERR_BUFFER_TOO_SMALL if smaller); it needs no initial
 * contents.  The call runs the kernel chain (never the persistent launch).
 *
 * hgd_decode_layer_stack_keep: stream b keeps the first keep[b] rows (int32 [B]
 * device, read on the device) of the verify call whose log is given: every GDN
 * layer's state takes those rows (hgd_gdn_keep), every conv tail takes their
 * inputs (hgd_conv1d_keep), and pos[b] += keep[b].  The state then equals the
 * state after keep[b] one-row decode calls on the same tokens, bit for bit.  A
 * keep[b] outside [0, T] leaves stream b as it is and writes
 * HGD_ERR_INVALID_ARG to *status_dev.  T must be the verify call's T. */
HGD_API int hgd_verify_log_bytes(const hgd_config* cfg, int B, int T, size_t* bytes);
HGD_API int hgd_decode_layer_stack_verify(const hgd_model* m, const hgd_state* st, const int32_t* tokens,
                                          int T, float* logits, int32_t* argmax, void* log,
                                          size_t log_bytes, int32_t* status_dev, hgd_stream_t stream);
HGD_API int hgd_decode_layer_stack_keep(const hgd_model* m, const hgd_state* st, int T, const void* log,
                                        size_t log_bytes, const int32_t* keep, int32_t* status_dev,
                                        hgd_stream_t stream);

/* Number of kernel launches one hgd_decode_layer_stack call over B streams and
 * T rows issues (-1 on bad arguments). */
HGD_API int hgd_decode_layer_stack_launches(const hgd_model* m, int B, int T);

/* ------------------------------------------------- tensor-core chain ---
 * [TF] PR body: windows of up to 16 rows of several streams per call, a
 * window's rows equal to one-row steps bit for bit.  A second decode path whose
 * projections are tcgen05 GEMMs (hgd_gemm_tc_bf16's kernel) over all of the
 * call's token rows: for windows of many rows the projections become dense
 * contractions that stream each weight once per call.  The tensor cores give a
 * token row the same bits whatever the number of rows in the call, and every
 * kernel between the GEMMs computes a row from that row's inputs alone, so a
 * window through this path equals its one-row steps through it bit for bit.
 * Its sums are ordered as the tensor cores order them, so it agrees with
 * hgd_decode_layer_stack (the mma.sync path) to fp32 rounding, not bit for bit:
 * decode a stream through one path.
 *
 * The weights, packed for the tensor cores, live in a second caller-owned
 * arena of hgd_model_tc_bytes bytes (256-byte aligned): fill it tensor by tensor
 * with hgd_model_tc_load from row-major bf16 copies (HGD_W_IN, HGD_W_OUT,
 * HGD_W_GATE, HGD_W_UP, HGD_W_DOWN per layer; layer -1: HGD_W_EMBED for the tied
 * head, HGD_W_LM_HEAD for an untied one), then hgd_model_attach_tc.  Requires
 * hidden, mlp_inter, the GDN and attention widths to be multiples of 64.
 * hgd_decode_layer_stack_tc: the arguments of hgd_decode_layer_stack; B*T up to
 * 256 rows; logits may be NULL (the state arena then holds them). */
HGD_API int hgd_model_tc_bytes(const hgd_config* cfg, size_t* bytes);
HGD_API int hgd_model_tc_load(const hgd_config* cfg, void* tc_arena, size_t bytes, int layer, int tensor,
                              const uint16_t* src, hgd_stream_t stream);
HGD_API int hgd_model_attach_tc(hgd_model* m, const void* tc_arena, size_t bytes);
HGD_API int hgd_decode_layer_stack_tc(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T,
                                      float* logits, int32_t* argmax, float* S_rec, float* tail_rec,
                                      int32_t* status_dev, hgd_stream_t stream);

/* ------------------------------------------------------ stack diagnostics --
 * The same check on the persistent decode launch itself ([LUCE] Known issues:
 * a grid-wide wait that can never complete deadlocks the whole kernel).  One
 * hgd_decode_layer_stack call over T rows that takes the persistent launch, in
 * which CTA `skip_cta` leaves out its arrival at the end of phase `skip_phase`
 * (phases count from 0: five per layer, then the LM head) and every phase wait
 * is limited to `wait_ms` (1..2000) instead of 2 s.  The waits for that phase
 * then run out: the kernel writes HGD_ERR_TIMEOUT to *status_dev (zero it
 * first), and every CTA skips the rest of the call, so the call ends.
 * report_dev (device uint32[4], 16-byte aligned, or NULL) receives what ran out
 * first {1 = a phase counter, 2 = a weight slab, 3 = a ring slot}, its phase,
 * the CTA that saw it, and 0.  The call leaves the state partly advanced (the
 * phases before the skipped arrival ran; positions do not advance) and argmax
 * unwritten: restore the state before decoding on.  HGD_ERR_UNSUPPORTED_SHAPE
 * if the call would not take the persistent launch. */
HGD_API int hgd_check_stack_timeout(const hgd_model* m, const hgd_state* st, const int32_t* tokens,
                                    int T, int32_t* argmax, int skip_cta, int skip_phase, int wait_ms,
                                    int32_t* status_dev, uint32_t* report_dev, hgd_stream_t stream);

/* The persistent launch's co-residency refusal: runs the host-side check that
 * precedes every persistent launch with the occupancy query's answer replaced
 * by zero resident CTAs per SM, and returns what hgd_decode_layer_stack returns
 * then (HGD_ERR_NOT_CORESIDENT).  Enqueues nothing. */
HGD_API int hgd_check_not_coresident(const hgd_model* m, const hgd_state* st, int T);

#ifdef __cplusplus
}
#endif
#endif /* HGD_H */
