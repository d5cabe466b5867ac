// gdn.cuh -- causal conv1d tail update and the gated-delta-rule state update.
//
// "qwen3_5 cuda: mixed-width MLX checkpoints ... #849", PR body: the gated delta
// rule and the causal convolution, windows of rows that record each row's
// recurrence and conv tail and equal one-row steps bit for bit.
// "Running on Turing (sm_75)", What was checked: GDN decode kernels keep the
// state [num_heads, V, K].
//
// State update per head, per row (beta, alpha scalars; k, q L2-normalised):
//   w_i = S_i . k,   delta_i = beta (v_i - alpha w_i),   S_i <- alpha S_i + delta_i k,
//   o_i = S_i . q
// which is S <- alpha S (I - beta k k^T) + beta v k^T, o = S q, written as a rank-1
// update so each of the dv rows of S is independent.  A warp owns RPW rows; lane
// l holds KPL consecutive k-elements of each row (a 16-byte load when KPL = 4),
// so every row of the fp32 state stays in registers across all T rows of a
// call and is read and written once per call.  The arithmetic of a row depends
// only on that row's inputs, so T-row calls equal T one-row calls bit for bit.
#pragma once

#include "common.cuh"

namespace hgd {

constexpr int GDN_WARPS = 4;
constexpr int GDN_RPW = 4;                        // state rows per warp
constexpr int GDN_ROWS = GDN_WARPS * GDN_RPW;     // state rows per CTA (16)

template <int KPL>
__device__ __forceinline__ void ld_vec(float (&d)[KPL], const float* p) {
    if (KPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    } else if (KPL == 8) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        const float4 u = *reinterpret_cast<const float4*>(p + 4);
        d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
        d[4] = u.x; d[5] = u.y; d[6] = u.z; d[7] = u.w;
    } else if (KPL == 2) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        d[0] = v.x; d[1] = v.y;
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e) d[e] = p[e];
    }
}
template <int KPL>
__device__ __forceinline__ void st_vec(float* p, const float (&d)[KPL]) {
    if (KPL == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(d[0], d[1], d[2], d[3]);
    } else if (KPL == 8) {
        *reinterpret_cast<float4*>(p) = make_float4(d[0], d[1], d[2], d[3]);
        *reinterpret_cast<float4*>(p + 4) = make_float4(d[4], d[5], d[6], d[7]);
    } else if (KPL == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(d[0], d[1]);
    } else {
#pragma unroll
        for (int e = 0; e < KPL; ++e) p[e] = d[e];
    }
}

// The rank-1 update of one state row by one logged row: S <- alpha S + delta k^T
// (the one expression both the step and the replay of a log use).
template <int KPL>
__device__ __forceinline__ void gdn_row_update(float (&S)[KPL], float delta, const float (&kv)[KPL], float alpha) {
#pragma unroll
    for (int e = 0; e < KPL; ++e) S[e] = fmaf(delta, kv[e], alpha * S[e]);
}

// One recurrent row for RPW state rows held by this warp.  kv/qv: this lane's
// normalised key/query elements; vrow[r]: value of state row r; returns o and
// the row's writes delta (every lane).  The RPW dot products of a kind are
// summed over the lanes together (warp_sum_transposed: warp_sum's pairings, so
// each sum is bitwise warp_sum's) and then broadcast.
template <int KPL, int RPW>
__device__ __forceinline__ void gdn_rows_step(float (&S)[RPW][KPL], const float (&kv)[KPL],
                                              const float (&qv)[KPL], float alpha, float beta,
                                              const float (&vrow)[RPW], float (&o)[RPW],
                                              float (&dl)[RPW]) {
    constexpr int LPR = 32 / RPW;  // lanes holding each sum after the transposed reduction
    const int lane = threadIdx.x & 31;
    float w[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        w[r] = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) w[r] = fmaf(S[r][e], kv[e], w[r]);
    }
    const float ws = warp_sum_transposed<RPW>(w, lane);
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const float delta = beta * (vrow[r] - alpha * __shfl_sync(0xffffffffu, ws, r * LPR));
        dl[r] = delta;
        gdn_row_update<KPL>(S[r], delta, kv, alpha);
    }
    float ov[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        ov[r] = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) ov[r] = fmaf(S[r][e], qv[e], ov[r]);
    }
    const float os = warp_sum_transposed<RPW>(ov, lane);
#pragma unroll
    for (int r = 0; r < RPW; ++r) o[r] = __shfl_sync(0xffffffffu, os, r * LPR);
}

// L2 normalisation scale 1/sqrt(sum x^2 + 1e-6) of a dk-vector held in shared
// memory, computed by one warp (lane-strided KPL chunks, then a butterfly).
template <int KPL>
__device__ __forceinline__ float l2_scale(const float* x, int lane) {
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
        const float a = x[lane * KPL + e];
        ss = fmaf(a, a, ss);
    }
    ss = warp_sum(ss);
    return rsqrtf(ss + 1e-6f);
}

// ------------------------------------------------------- standalone GDN step
struct GdnParams {
    const float* q; const float* k; const float* v; int64_t stride;
    const float* g; const float* b;
    float* S; float* o; bf16_t* o_bf16; float* S_rec;
    int B, T, H, dk, dv, l2norm;
    int grp;  // value heads per query/key head: value head h reads q, k of head h / grp
};

// grid (B*H, dv/16), block 128: a CTA owns 16 state rows of one (stream, head).
template <int KPL>
__global__ void __launch_bounds__(GDN_WARPS * 32) k_gdn_step(const __grid_constant__ GdnParams p) {
    pdl_launch();
    pdl_wait();
    constexpr int DK = 32 * KPL;
    __shared__ float qs[DK], ks[DK], coef[4];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int row0 = blockIdx.y * GDN_ROWS + warp * GDN_RPW;
    float S[GDN_RPW][KPL];
    float* Sbase = p.S + ((int64_t)(b * p.H + h) * p.dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);

    for (int t = 0; t < p.T; ++t) {
        const int64_t row = (int64_t)b * p.T + t;
        const float* qp = p.q + row * p.stride + (int64_t)(h / p.grp) * DK;
        const float* kp = p.k + row * p.stride + (int64_t)(h / p.grp) * DK;
        __syncthreads();
        for (int i = tid; i < DK; i += GDN_WARPS * 32) { qs[i] = qp[i]; ks[i] = kp[i]; }
        __syncthreads();
        if (warp == 0) { const float s = p.l2norm ? l2_scale<KPL>(qs, lane) : 1.f; if (lane == 0) coef[0] = s; }
        if (warp == 1) { const float s = p.l2norm ? l2_scale<KPL>(ks, lane) : 1.f; if (lane == 0) coef[1] = s; }
        if (warp == 2 && lane == 0) {
            coef[2] = expf(p.g[row * p.H + h]);
            coef[3] = sigmoid_f(p.b[row * p.H + h]);
        }
        __syncthreads();
        float kv[KPL], qv[KPL];
#pragma unroll
        for (int e = 0; e < KPL; ++e) { qv[e] = qs[lane * KPL + e] * coef[0]; kv[e] = ks[lane * KPL + e] * coef[1]; }
        float vrow[GDN_RPW], o[GDN_RPW], dl[GDN_RPW];
        const float* vp = p.v + row * p.stride + (int64_t)h * p.dv + row0;
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) vrow[r] = vp[r];
        gdn_rows_step<KPL>(S, kv, qv, coef[2], coef[3], vrow, o, dl);
        const int64_t orow = (row * p.H + h) * p.dv + row0;
        if (lane < GDN_RPW) {
            float ov = o[0];
#pragma unroll
            for (int r = 1; r < GDN_RPW; ++r) if (lane == r) ov = o[r];
            p.o[orow + lane] = ov;
            if (p.o_bf16) p.o_bf16[orow + lane] = f2bf(ov);
        }
        if (p.S_rec) {
            float* rp = p.S_rec + ((row * p.H + h) * p.dv + row0) * DK + lane * KPL;
#pragma unroll
            for (int r = 0; r < GDN_RPW; ++r) st_vec<KPL>(rp + (int64_t)r * DK, S[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) st_vec<KPL>(Sbase + (int64_t)r * DK, S[r]);
}

// ------------------------------------------------- recurrence logs and keep
// "qwen3_5 cuda ... #849", tree-window commit note: a verify window logs each
// row's decay, write and key instead of snapshotting the state, and keep replays
// the kept rows onto the recurrence in one pass.  The window kernel runs the
// step's arithmetic on the state held in registers and never stores it; the
// keep kernel applies the logged (alpha, delta, k) with the step's own update
// expression, so keep(n) equals n one-row steps bit for bit.
struct GdnLogParams {
    const float* q; const float* k; const float* v; int64_t stride;
    const float* g; const float* b;
    const float* S; float* o; bf16_t* o_bf16;
    float* log_alpha; float* log_delta; float* log_k;   // [B,T,H], [B,T,H,dv], [B,T,H,dk]
    int B, T, H, dk, dv, l2norm;
    int grp;  // value heads per query/key head
};

// grid (B*H, dv/16), block 128, as k_gdn_step.
template <int KPL>
__global__ void __launch_bounds__(GDN_WARPS * 32) k_gdn_window_log(const __grid_constant__ GdnLogParams p) {
    pdl_launch();
    pdl_wait();
    constexpr int DK = 32 * KPL;
    __shared__ float qs[DK], ks[DK], coef[4];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int row0 = blockIdx.y * GDN_ROWS + warp * GDN_RPW;
    float S[GDN_RPW][KPL];
    const float* Sbase = p.S + ((int64_t)(b * p.H + h) * p.dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);

    for (int t = 0; t < p.T; ++t) {
        const int64_t row = (int64_t)b * p.T + t;
        const float* qp = p.q + row * p.stride + (int64_t)(h / p.grp) * DK;
        const float* kp = p.k + row * p.stride + (int64_t)(h / p.grp) * DK;
        __syncthreads();
        for (int i = tid; i < DK; i += GDN_WARPS * 32) { qs[i] = qp[i]; ks[i] = kp[i]; }
        __syncthreads();
        if (warp == 0) { const float s = p.l2norm ? l2_scale<KPL>(qs, lane) : 1.f; if (lane == 0) coef[0] = s; }
        if (warp == 1) { const float s = p.l2norm ? l2_scale<KPL>(ks, lane) : 1.f; if (lane == 0) coef[1] = s; }
        if (warp == 2 && lane == 0) {
            coef[2] = expf(p.g[row * p.H + h]);
            coef[3] = sigmoid_f(p.b[row * p.H + h]);
        }
        __syncthreads();
        float kv[KPL], qv[KPL];
#pragma unroll
        for (int e = 0; e < KPL; ++e) { qv[e] = qs[lane * KPL + e] * coef[0]; kv[e] = ks[lane * KPL + e] * coef[1]; }
        float vrow[GDN_RPW], o[GDN_RPW], dl[GDN_RPW];
        const float* vp = p.v + row * p.stride + (int64_t)h * p.dv + row0;
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) vrow[r] = vp[r];
        gdn_rows_step<KPL>(S, kv, qv, coef[2], coef[3], vrow, o, dl);
        const int64_t orow = (row * p.H + h) * p.dv + row0;
        if (lane < GDN_RPW) {
            float ov = o[0], dv_ = dl[0];
#pragma unroll
            for (int r = 1; r < GDN_RPW; ++r) if (lane == r) { ov = o[r]; dv_ = dl[r]; }
            p.o[orow + lane] = ov;
            if (p.o_bf16) p.o_bf16[orow + lane] = f2bf(ov);
            p.log_delta[orow + lane] = dv_;
        }
        if (blockIdx.y == 0 && warp == 0) {
            st_vec<KPL>(p.log_k + (row * p.H + h) * DK + lane * KPL, kv);
            if (lane == 0) p.log_alpha[row * p.H + h] = coef[2];
        }
    }
}

struct GdnKeepParams {
    float* S; const float* log_alpha; const float* log_delta; const float* log_k;
    const int32_t* keep; int32_t* status;
    int B, T, H, dv;
};

// grid (B*H, dv/16), block 128: the CTA's 16 state rows of one (stream, head)
// take the stream's first keep[b] logged rows.  A count outside [0, T] leaves
// the stream's state as it is and reports HGD_ERR_INVALID_ARG.
template <int KPL>
__global__ void __launch_bounds__(GDN_WARPS * 32) k_gdn_keep(const __grid_constant__ GdnKeepParams p) {
    pdl_launch();
    pdl_wait();
    constexpr int DK = 32 * KPL;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int row0 = blockIdx.y * GDN_ROWS + warp * GDN_RPW;
    const int n = p.keep[b];
    if (n < 0 || n > p.T) {
        if (h == 0 && blockIdx.y == 0 && tid == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
        return;
    }
    if (n == 0) return;
    float S[GDN_RPW][KPL];
    float* Sbase = p.S + ((int64_t)(b * p.H + h) * p.dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);
    for (int t = 0; t < n; ++t) {
        const int64_t lr = ((int64_t)b * p.T + t) * p.H + h;
        const float alpha = p.log_alpha[lr];
        float kv[KPL], dl[GDN_RPW];
        ld_vec<KPL>(kv, p.log_k + lr * DK + lane * KPL);
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) dl[r] = p.log_delta[lr * p.dv + row0 + r];
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) gdn_row_update<KPL>(S[r], dl[r], kv, alpha);
    }
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) st_vec<KPL>(Sbase + (int64_t)r * DK, S[r]);
}

// The conv tail after the first keep[b] rows of a window: one thread per
// (stream, channel) shifts in x rows 0..keep[b]-1 (the copies the stepped conv
// makes).  A count outside [0, T] leaves the stream's tail and reports
// HGD_ERR_INVALID_ARG.
struct ConvKeepParams {
    float* tail; const float* x; const int32_t* keep; int32_t* status;
    int B, T, C, kc;
};
__global__ void k_conv_keep(const __grid_constant__ ConvKeepParams p) {
    pdl_launch();
    pdl_wait();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.B * p.C) return;
    const int b = (int)(idx / p.C), c = (int)(idx % p.C);
    const int n = p.keep[b], nt = p.kc - 1;
    if (n < 0 || n > p.T) {
        if (c == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
        return;
    }
    float tl[8];
    float* tb = p.tail + (int64_t)b * nt * p.C + c;
    for (int j = 0; j < nt; ++j) tl[j] = tb[(int64_t)j * p.C];
    for (int t = 0; t < n; ++t) {
        const float xv = p.x[((int64_t)b * p.T + t) * p.C + c];
        for (int j = 0; j + 1 < nt; ++j) tl[j] = tl[j + 1];
        if (nt > 0) tl[nt - 1] = xv;
    }
    for (int j = 0; j < nt; ++j) tb[(int64_t)j * p.C] = tl[j];
}

// ---------------------------------------------------------- standalone conv
struct ConvParams {
    const float* x; float* tail; const bf16_t* w; float* y; float* tail_rec;
    int B, T, C, kc, silu;
};

// One thread per (stream, channel); rows in order.
__global__ void k_conv_tail(const __grid_constant__ ConvParams p) {
    pdl_launch();
    pdl_wait();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.B * p.C) return;
    const int b = (int)(idx / p.C), c = (int)(idx % p.C);
    const int nt = p.kc - 1;
    float tl[8], w[8];
    for (int j = 0; j < p.kc; ++j) w[j] = bf2f(p.w[(int64_t)c * p.kc + j]);
    float* tb = p.tail + (int64_t)b * nt * p.C + c;
    for (int j = 0; j < nt; ++j) tl[j] = tb[(int64_t)j * p.C];
    for (int t = 0; t < p.T; ++t) {
        const int64_t row = (int64_t)b * p.T + t;
        const float xv = p.x[row * p.C + c];
        float s = 0.f;
        for (int j = 0; j < nt; ++j) s = fmaf(w[j], tl[j], s);
        s = fmaf(w[nt], xv, s);
        p.y[row * p.C + c] = p.silu ? silu_f(s) : s;
        for (int j = 0; j + 1 < nt; ++j) tl[j] = tl[j + 1];
        if (nt > 0) tl[nt - 1] = xv;
        if (p.tail_rec)
            for (int j = 0; j < nt; ++j) p.tail_rec[(row * nt + j) * p.C + c] = tl[j];
    }
    for (int j = 0; j < nt; ++j) tb[(int64_t)j * p.C] = tl[j];
}

// ------------------------------------------------------- stack: GDN mixer
// Gates from a/b, L2 norm and the state update of one GDN layer of the stack.
// The projection rows already hold the conv outputs of the q|k|v channels (the
// conv runs in the in-projection's epilogue).  grid (B*H, dv/16), block 128.
// Rows (b, t) are token rows b*T + t of the projection buffer [M][proj_ld] with
// columns q (H*dk) | k (H*dk) | v (H*dv) | z (H*dv) | a (H) | b (H).
struct GdnLayerParams {
    const float* proj; int64_t proj_ld;
    const bf16_t* A_log; const bf16_t* dt_bias;  // [H]
    float* S;                   // this layer: [B][H][dv][dk]
    float* o; int64_t o_ld;     // [M][o_ld]
    float* S_rec;               // this layer: [B][T][H][dv][dk] or null
    // a verify window's logs ([B][T][H], [B][T][H][dv], [B][T][H][dk]) or null;
    // when set, the rows run on the state in registers and S is not written back
    float* log_alpha; float* log_delta; float* log_k;
    int B, T, H, dv;
    int Hk;  // query/key heads (H, the value heads, is a multiple): value head h reads head h / (H / Hk)
    // the fused gated RMSNorm (k_gdn_layer<.., GN = true>, one CTA per (stream, head)):
    // z rows, the norm gains and the output rows packed for the tensor-core GEMM
    const float* z; int64_t z_ld; const bf16_t* gn_w; bf16_t* u; int u_ntp; float eps;
    // the fused causal conv (CONV = true, with GN and H = Hk): this layer's tails
    // [B][kc-1][C], the conv weights [C][kc], tail records [B][T][kc-1][C] or null,
    // and the conv channel count C; proj then holds the raw in-projection rows
    float* conv_tail; const bf16_t* conv_w; float* conv_tail_rec; int C;
};
constexpr int GDN_CONV_K = 4;  // the causal conv's width

// Rows whose inputs k_gdn_layer stages in shared memory at once.
constexpr int GDN_TB = 16;

// RPW: state rows per warp (4 or 8; the per-row arithmetic does not depend on it);
// NW warps per CTA.  GN: the CTA holds all dv rows of its head (NW * RPW = dv,
// one CTA per (stream, head)) and forms the gated RMSNorm of the rows' outputs
// itself (gated_norm_warp, the arithmetic of k_gated_norm) into p.u, instead of
// writing o.
// CONV (with GN, H = Hk): the CTA also runs the causal conv of its head's q, k and
// v channels (one thread per channel, rows in order, the arithmetic of k_tc_conv)
// on the staged raw rows, so no separate conv pass runs.
template <int KPL, int RPW, int NW = GDN_WARPS, bool GN = false, bool CONV = false>
__global__ void __launch_bounds__(NW * 32) k_gdn_layer(const __grid_constant__ GdnLayerParams p) {
    pdl_launch();
    pdl_wait();
    constexpr int DK = 32 * KPL, NT = NW * 32, ROWS = NW * RPW;
    __shared__ float os[GN ? GDN_TB : 1][GN ? ROWS : 1];  // GN: the block's output rows
    // A block of up to GDN_TB rows at a time: every input of the block (q and k
    // of the key head, this CTA's value rows, a and b) is loaded in one batch,
    // the rows' L2 scales and gates are formed in parallel, and then only the
    // recurrence runs row after row, from shared memory, with no barrier.  Each
    // value comes from the function the one-row kernels use (l2_scale, the gate
    // expressions, gdn_rows_step), so the results are theirs bit for bit.
    __shared__ __align__(16) float qs[GDN_TB][DK], ks[GDN_TB][DK], vs[GDN_TB][ROWS];
    __shared__ float qsc[GDN_TB], ksc[GDN_TB], al[GDN_TB], be[GDN_TB];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H, dv = p.dv;
    const int b = blockIdx.x / H, h = blockIdx.x % H;
    const int row0 = blockIdx.y * ROWS + warp * RPW;
    const int Hk = p.Hk, hk = h / (H / Hk);
    const int64_t C = 2 * (int64_t)Hk * DK + (int64_t)H * dv;
    const float A = expf(bf2f(p.A_log[h])), dtb = bf2f(p.dt_bias[h]);

    // CONV: this thread's channel (q, k, then v channels of the head), its weights
    // and tail, in registers for the whole call
    constexpr int NT3 = GDN_CONV_K - 1;
    static_assert(!CONV || (GN && 2 * DK + ROWS <= NT), "one thread per conv channel");
    int cch = -1;
    float cw[GDN_CONV_K], ctl[NT3];
    if (CONV && tid < 2 * DK + ROWS) {
        cch = tid < DK ? hk * DK + tid
                       : tid < 2 * DK ? Hk * DK + hk * DK + (tid - DK) : 2 * Hk * DK + h * dv + (tid - 2 * DK);
#pragma unroll
        for (int j = 0; j < GDN_CONV_K; ++j) cw[j] = bf2f(p.conv_w[(int64_t)cch * GDN_CONV_K + j]);
#pragma unroll
        for (int j = 0; j < NT3; ++j) ctl[j] = p.conv_tail[((int64_t)b * NT3 + j) * p.C + cch];
    }

    float S[RPW][KPL];
    float* Sbase = p.S + ((int64_t)(b * H + h) * dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);

    __shared__ float abr[2][GDN_TB];  // raw a and b of the block's rows
    // rows start on 16-byte boundaries (q and k heads are multiples of 32 floats)
    const bool v16 = (p.proj_ld & 3) == 0 && (reinterpret_cast<uintptr_t>(p.proj) & 15) == 0;
    for (int t0 = 0; t0 < p.T; t0 += GDN_TB) {
        const int n = min(GDN_TB, p.T - t0);
        const float* pr0 = p.proj + ((int64_t)b * p.T + t0) * p.proj_ld;
        // the block's inputs straight into shared memory (cp.async): q and k in
        // 16-byte pieces, this CTA's value rows, a and b
        if (v16) {
            for (int i = tid; i < n * (DK / 4); i += NT) {
                const int t = i / (DK / 4), e = (i % (DK / 4)) * 4;
                const float* pr = pr0 + (int64_t)t * p.proj_ld;
                cp_async16(&qs[t][e], pr + (int64_t)hk * DK + e);
                cp_async16(&ks[t][e], pr + (int64_t)Hk * DK + (int64_t)hk * DK + e);
            }
        } else {
            for (int i = tid; i < n * DK; i += NT) {
                const int t = i / DK, e = i % DK;
                const float* pr = pr0 + (int64_t)t * p.proj_ld;
                cp_async4(&qs[t][e], pr + (int64_t)hk * DK + e);
                cp_async4(&ks[t][e], pr + (int64_t)Hk * DK + (int64_t)hk * DK + e);
            }
        }
        for (int i = tid; i < n * ROWS; i += NT) {
            const int t = i / ROWS, r = i % ROWS;
            cp_async4(&vs[t][r], pr0 + (int64_t)t * p.proj_ld + 2 * (int64_t)Hk * DK + (int64_t)h * dv +
                                     blockIdx.y * ROWS + r);
        }
        if (tid < n) {
            cp_async4(&abr[0][tid], pr0 + (int64_t)tid * p.proj_ld + C + (int64_t)H * dv + h);
            cp_async4(&abr[1][tid], pr0 + (int64_t)tid * p.proj_ld + C + (int64_t)H * dv + H + h);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
        if (CONV) {
            if (cch >= 0) {
                float* col = tid < DK ? &qs[0][tid] : tid < 2 * DK ? &ks[0][tid - DK] : &vs[0][tid - 2 * DK];
                const int stride = tid < 2 * DK ? DK : ROWS;
                for (int t = 0; t < n; ++t) {
                    const float xv = col[t * stride];
                    float acc = 0.f;
#pragma unroll
                    for (int j = 0; j < NT3; ++j) acc = fmaf(cw[j], ctl[j], acc);
                    acc = fmaf(cw[NT3], xv, acc);
                    col[t * stride] = silu_f(acc);
#pragma unroll
                    for (int j = 0; j + 1 < NT3; ++j) ctl[j] = ctl[j + 1];
                    ctl[NT3 - 1] = xv;
                    if (p.conv_tail_rec) {
                        float* rp = p.conv_tail_rec + ((int64_t)b * p.T + t0 + t) * NT3 * p.C + cch;
#pragma unroll
                        for (int j = 0; j < NT3; ++j) rp[(int64_t)j * p.C] = ctl[j];
                    }
                }
            }
            __syncthreads();
        }
        if (tid < n) {
            al[tid] = expf(-A * softplus_f(abr[0][tid] + dtb));
            be[tid] = sigmoid_f(abr[1][tid]);
        }
        for (int t = warp; t < n; t += NW) {
            const float a = l2_scale<KPL>(qs[t], lane), c = l2_scale<KPL>(ks[t], lane);
            if (lane == 0) { qsc[t] = a; ksc[t] = c; }
        }
        __syncthreads();
        for (int t = 0; t < n; ++t) {
            const int64_t row = (int64_t)b * p.T + t0 + t;
            const float qa = qsc[t], ka = ksc[t], alpha = al[t], beta = be[t];
            float kv[KPL], qv[KPL], vrow[RPW];
#pragma unroll
            for (int e = 0; e < KPL; ++e) { qv[e] = qs[t][lane * KPL + e] * qa; kv[e] = ks[t][lane * KPL + e] * ka; }
#pragma unroll
            for (int r = 0; r < RPW; ++r) vrow[r] = vs[t][warp * RPW + r];
            float o[RPW], dl[RPW];
            gdn_rows_step<KPL, RPW>(S, kv, qv, alpha, beta, vrow, o, dl);
            if (lane < RPW) {
                float ov = o[0], dv_ = dl[0];
#pragma unroll
                for (int r = 1; r < RPW; ++r) if (lane == r) { ov = o[r]; dv_ = dl[r]; }
                if (GN) os[t][warp * RPW + lane] = ov;
                else p.o[row * p.o_ld + (int64_t)h * dv + row0 + lane] = ov;
                if (p.log_delta) p.log_delta[(row * H + h) * dv + row0 + lane] = dv_;
            }
            if (p.log_delta && blockIdx.y == 0 && warp == 0) {
                st_vec<KPL>(p.log_k + (row * H + h) * DK + lane * KPL, kv);
                if (lane == 0) p.log_alpha[row * H + h] = alpha;
            }
            if (p.S_rec) {
                float* rp = p.S_rec + ((row * H + h) * dv + row0) * DK + lane * KPL;
#pragma unroll
                for (int r = 0; r < RPW; ++r) st_vec<KPL>(rp + (int64_t)r * DK, S[r]);
            }
        }
        if (GN) {
            __syncthreads();
            for (int t = warp; t < n; t += NW) {
                const int64_t row = (int64_t)b * p.T + t0 + t;
                gated_norm_warp(os[t], p.z + row * p.z_ld + (int64_t)h * dv, p.gn_w, dv, p.eps, lane,
                                [&](int i, bf16_t v) { p.u[tc_x_elem((int)row, h * dv + i, p.u_ntp)] = v; });
            }
        }
        __syncthreads();  // the next block's inputs overwrite these
    }
    if (p.log_delta) return;  // a verify window: the state stays as it was
#pragma unroll
    for (int r = 0; r < RPW; ++r) st_vec<KPL>(Sbase + (int64_t)r * DK, S[r]);
    if (CONV && cch >= 0)
#pragma unroll
        for (int j = 0; j < NT3; ++j) p.conv_tail[((int64_t)b * NT3 + j) * p.C + cch] = ctl[j];
}

}  // namespace hgd
