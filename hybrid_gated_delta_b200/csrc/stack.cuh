// stack.cuh -- one cooperative launch for a whole decode step of the stack.
//
// "luce-megakernel HANDOFF.md", Architecture: all 24 layers of the decode step
// in one persistent kernel with grid synchronisation between layers (and its
// Known Issues: a grid sync deadlocks unless every block is resident, hence a
// cooperative launch).  Built for B200 here:
//  * one CTA per SM: a producer warp and eight consumer warps;
//  * the producer walks the CTA's share of every projection of the step, in
//    order, and streams each 16-row x 256-column weight slab (8 KB, contiguous
//    thanks to the fragment-ordered packing) with one bulk copy (cp.async.bulk,
//    no multicast, L2 evict-first) into the two-slot ring of the consumer warp
//    that owns it, feeding the warps slab by slab in turn.  Weights never depend
//    on activations, so it runs ahead across phase boundaries and keeps HBM busy
//    while the consumers wait at a grid barrier.  Each warp waits on its own
//    slots strictly in order, so an mbarrier phase parity never aliases;
//  * the consumers run the phases in order -- per GDN layer: in-projection with
//    the fused causal conv, gated delta rule, out-projection with the gated
//    RMSNorm, SwiGLU, down-projection; per attention layer: in-projection, RoPE
//    and KV append, attention partials, merge, out-projection, SwiGLU, down; then
//    the LM head with the argmax -- and meet at a grid barrier after each;
//  * every phase runs the same per-row arithmetic as the per-kernel path (the
//    same device functions, the same slab order), so the two agree bit for bit;
//  * every wait is bounded; a wait that runs out sets HGD_ERR_TIMEOUT and a
//    global abort flag, after which every CTA skips the remaining work.
#pragma once

#include "attn.cuh"
#include "gdn.cuh"
#include "gemv.cuh"

namespace hgd {

constexpr int SK_CW = 8;                        // consumer warps
constexpr int SK_THREADS = (SK_CW + 1) * 32;    // + the producer warp
constexpr int SK_SLAB_BYTES = GV_SLAB_STEPS * 1024;
constexpr int SK_NSW = 2;                       // ring slots per consumer warp
constexpr int SK_NSLOT = SK_CW * SK_NSW;        // 16 slots (128 KB)
constexpr int SK_MAXM = 8;                      // token rows per call (one MMA n-tile)

enum SkKind { SK_IN_GDN = 0, SK_GDN, SK_OUT_GDN, SK_IN_ATT, SK_ROPE, SK_PART, SK_MERGE, SK_OUT_ATT, SK_SWIGLU,
              SK_DOWN, SK_HEAD, SK_FINAL };

struct SkLayer { const bf16_t* w[HGD_W_LAYER_COUNT]; };

struct SkParams {
    int L, D, V, H, dk, dv, nq, nkv, hd, I, every;
    int C, gdn_out, attn_out, proj_ld;
    float eps, rope_base;
    int B, T, M, Lmax, max_chunks;
    const bf16_t* embed; const bf16_t* final_norm;
    float* S; float* conv; bf16_t* kv; int32_t* pos;
    bf16_t* resid; float* proj; float* obuf; float* qrot; bf16_t* attn; float* part; bf16_t* mlp;
    float* bestv; int32_t* besti; float* ws_part; int32_t* ws_cnt;
    const int32_t* tokens; float* logits; int32_t* argmax; float* S_rec; float* tail_rec;
    int32_t* status;
    unsigned* bar;   // [0] arrivals, [1] generation, [2] abort, [4..13] where the first wait ran out
    unsigned long long* trace;  // %globaltimer at the start of each phase (CTA 0), or null
    int x_bytes;
    SkLayer layer[HGD_MAX_LAYERS];
};

__device__ __forceinline__ bool sk_attn(const SkParams& s, int l) { return l % s.every == s.every - 1; }
__device__ __forceinline__ int sk_nphase(const SkParams& s, int l) { return sk_attn(s, l) ? 7 : 5; }
__device__ __forceinline__ int sk_kind(const SkParams& s, int l, int j) {
    if (l == s.L) return j == 0 ? SK_HEAD : SK_FINAL;
    static constexpr int gdn[5] = {SK_IN_GDN, SK_GDN, SK_OUT_GDN, SK_SWIGLU, SK_DOWN};
    static constexpr int att[7] = {SK_IN_ATT, SK_ROPE, SK_PART, SK_MERGE, SK_OUT_ATT, SK_SWIGLU, SK_DOWN};
    return sk_attn(s, l) ? att[j] : gdn[j];
}
__device__ __forceinline__ bool sk_is_gemv(int k) {
    return k == SK_IN_GDN || k == SK_OUT_GDN || k == SK_IN_ATT || k == SK_OUT_ATT || k == SK_SWIGLU ||
           k == SK_DOWN || k == SK_HEAD;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Record the first wait that ran out (what: 1 grid barrier, 2 weight slab,
// 3 free ring slot) with its phase, CTA and ring sequence number; set the
// status and the global abort flag.
__device__ __forceinline__ void sk_timeout(unsigned* bar, int32_t* status, unsigned what, unsigned phase,
                                           unsigned seq) {
    if (atomicCAS(&bar[4], 0u, what) == 0u) {
        bar[5] = phase;
        bar[6] = blockIdx.x;
        bar[7] = seq;
    }
    set_status(status, HGD_ERR_TIMEOUT);
    atomicExch(&bar[2], 1u);
}

// The GEMV of a phase.  Row blocks below 2 per CTA split their slabs over CTAs.
__device__ __forceinline__ void sk_gemv_params(const SkParams& s, int kind, int l, int ig, GemvParams& p) {
    p = GemvParams{};
    const bf16_t* const* w = l < s.L ? s.layer[l].w : nullptr;
    p.packed = 1;
    p.M = s.M;
    p.eps = s.eps;
    p.status = s.status;
    const size_t c_layer = (size_t)s.B * (GV_CONV_K - 1) * s.C;
    const size_t trec_layer = (size_t)s.B * s.T * (GV_CONV_K - 1) * s.C;
    bool swi = false;
    switch (kind) {
        case SK_IN_GDN: case SK_IN_ATT:
            p.W = w[HGD_W_IN]; p.N = kind == SK_IN_GDN ? s.gdn_out : s.attn_out; p.K = s.D;
            p.x = s.resid; p.x_ld = s.D; p.norm_w = w[HGD_W_IN_NORM];
            p.y = s.proj; p.y_ld = s.proj_ld;
            if (l == 0) { p.tokens = s.tokens; p.embed = s.embed; p.vocab = s.V; p.resid_out = s.resid; p.resid_out_ld = s.D; }
            if (kind == SK_IN_GDN) {
                p.conv_w = w[HGD_W_CONV]; p.conv_tail = s.conv + ig * c_layer;
                p.conv_rec = s.tail_rec ? s.tail_rec + ig * trec_layer : nullptr;
                p.conv_C = s.C; p.conv_T = s.T; p.m0 = 0;
            }
            break;
        case SK_OUT_GDN:
            p.W = w[HGD_W_OUT]; p.N = s.D; p.K = s.H * s.dv;
            p.o = s.obuf; p.o_ld = (int64_t)s.H * s.dv; p.z = s.proj + s.C; p.z_ld = s.proj_ld;
            p.gnorm_w = w[HGD_W_GNORM]; p.gn_d = s.dv;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        case SK_OUT_ATT:
            p.W = w[HGD_W_OUT]; p.N = s.D; p.K = s.nq * s.hd;
            p.x = s.attn; p.x_ld = (int64_t)s.nq * s.hd;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        case SK_SWIGLU:
            p.W = w[HGD_W_GATE]; p.N = s.I; p.K = s.D; swi = true;
            p.x = s.resid; p.x_ld = s.D; p.norm_w = w[HGD_W_POST_NORM];
            p.y = s.mlp; p.y_ld = s.I;
            break;
        case SK_DOWN:
            p.W = w[HGD_W_DOWN]; p.N = s.D; p.K = s.I;
            p.x = s.mlp; p.x_ld = s.I;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        default:  // SK_HEAD
            p.W = s.embed; p.N = s.V; p.K = s.D;
            p.x = s.resid; p.x_ld = s.D; p.norm_w = s.final_norm;
            p.logits = s.logits; p.logits_ld = s.V; p.best_v = s.bestv; p.best_i = s.besti;
            break;
    }
    p.nks = gv_slabs(p.K);
    p.n_rowblk = swi ? (p.N + 7) / 8 : (p.N + GV_ROWS - 1) / GV_ROWS;
    p.split = (kind != SK_HEAD && p.n_rowblk < 2 * (int)gridDim.x) ? 1 : 0;
    p.n_items = p.n_rowblk * (p.split ? p.nks : 1);
    if (p.split) { p.ws_part = s.ws_part; p.ws_cnt = s.ws_cnt; p.ws_mp = 8; }
    p.x_bytes = s.x_bytes;
}

// Items of this CTA in a phase of n items: c, c + G, c + 2G, ...
__device__ __forceinline__ int sk_cta_items(int n) {
    const int c = blockIdx.x, G = gridDim.x;
    return c < n ? (n - c + G - 1) / G : 0;
}

// Grid barrier among the consumer warps of all CTAs (the producer warps do not
// take part).  Returns false if the wait ran out or an abort was raised.
__device__ bool sk_grid_sync(const SkParams& s, volatile int* cta_abort, int phase) {
    named_bar(1, SK_CW * 32);
    if (threadIdx.x == 0) {
        bool ok = !*cta_abort;
        __threadfence();
        const unsigned gen = ld_acquire_u32(&s.bar[1]);
        const unsigned arrived = atomicAdd(&s.bar[0], 1u);
        if (arrived == gridDim.x - 1) {
            atomicExch(&s.bar[0], 0u);
            __threadfence();
            atomicAdd(&s.bar[1], 1u);
        } else {
            const unsigned long long t0 = globaltimer();
            while (ld_acquire_u32(&s.bar[1]) == gen) {
                if (ld_acquire_u32(&s.bar[2])) { ok = false; break; }
                if (globaltimer() - t0 > kWaitLimitNs) {
                    sk_timeout(s.bar, s.status, 1u, (unsigned)phase, arrived);
                    ok = false;
                    break;
                }
            }
        }
        __threadfence();
        if (!ok) *cta_abort = 1;
    }
    named_bar(1, SK_CW * 32);
    return !*cta_abort;
}

// ------------------------------------------------------------ non-GEMV items

// Gated delta rule for the 4 state rows row0..row0+3 (one warp) of stream b,
// head h of GDN layer l (index ig), over the call's T rows.  The arithmetic of
// every row is that of k_gdn_layer: the same norms, gates and gdn_rows_step.
template <int KPL>
__device__ void sk_gdn_item(const SkParams& s, int l, int ig, int b, int h, int row0, int lane) {
    constexpr int DK = 32 * KPL;
    const int H = s.H, dv = s.dv;
    const bf16_t* const* w = s.layer[l].w;
    const float A = expf(bf2f(w[HGD_W_A_LOG][h])), dtb = bf2f(w[HGD_W_DT_BIAS][h]);
    float S[GDN_RPW][KPL];
    float* Sbase = s.S + (size_t)ig * s.B * H * dv * DK + ((int64_t)(b * H + h) * dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);
    for (int t = 0; t < s.T; ++t) {
        const int64_t row = (int64_t)b * s.T + t;
        const float* pr = s.proj + row * s.proj_ld;
        float qv[KPL], kv[KPL];
        ld_vec<KPL>(qv, pr + (int64_t)h * DK + lane * KPL);
        ld_vec<KPL>(kv, pr + (int64_t)H * DK + (int64_t)h * DK + lane * KPL);
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) { sq = fmaf(qv[e], qv[e], sq); sk = fmaf(kv[e], kv[e], sk); }
        const float qsc = rsqrtf(warp_sum(sq) + 1e-6f), ksc = rsqrtf(warp_sum(sk) + 1e-6f);
#pragma unroll
        for (int e = 0; e < KPL; ++e) { qv[e] = qv[e] * qsc; kv[e] = kv[e] * ksc; }
        const float a = pr[s.C + (int64_t)H * dv + h];
        const float braw = pr[s.C + (int64_t)H * dv + H + h];
        const float alpha = expf(-A * softplus_f(a + dtb));
        const float beta = sigmoid_f(braw);
        float vrow[GDN_RPW], o[GDN_RPW];
        const float* vp = pr + 2 * (int64_t)H * DK + (int64_t)h * dv + row0;
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) vrow[r] = vp[r];
        gdn_rows_step<KPL>(S, kv, qv, alpha, beta, vrow, o);
        if (lane < GDN_RPW) {
            float ov = o[0];
#pragma unroll
            for (int r = 1; r < GDN_RPW; ++r) if (lane == r) ov = o[r];
            s.obuf[row * ((int64_t)H * dv) + (int64_t)h * dv + row0 + lane] = ov;
        }
        if (s.S_rec) {
            float* rp = s.S_rec + (size_t)ig * s.B * s.T * H * dv * DK +
                        ((((int64_t)b * s.T + t) * H + h) * dv + row0) * DK + lane * KPL;
#pragma unroll
            for (int r = 0; r < GDN_RPW; ++r) st_vec<KPL>(rp + (int64_t)r * DK, S[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) st_vec<KPL>(Sbase + (int64_t)r * DK, S[r]);
}

// RoPE of one head of one row (query heads: rotated q; key/value heads: the
// rotated key and the value appended to the cache), as k_rope_append computes it.
__device__ void sk_rope_item(const SkParams& s, int ia, int row, int head, int lane) {
    const int b = row / s.T, t = row % s.T;
    const int P = s.pos[b] + t;
    if (P < 0 || P >= s.Lmax) {
        if (lane == 0) set_status(s.status, HGD_ERR_INVALID_ARG);
        return;
    }
    const int hd = s.hd, half = hd / 2, qw = s.nq * hd;
    const float* pr = s.proj + (int64_t)row * s.proj_ld;
    const size_t kv_half = (size_t)s.B * s.nkv * s.Lmax * hd;
    bf16_t* kc = s.kv + (size_t)ia * 2 * kv_half;
    bf16_t* vc = kc + kv_half;
    for (int i = lane; i < half; i += 32) {
        const double inv = exp2(-2.0 * (double)i / (double)hd * log2((double)s.rope_base));
        const double th = (double)P * inv;
        const double tw = 6.283185307179586476925286766559;
        const float r = (float)(th - tw * rint(th / tw));
        float sn, cs;
        sincosf(r, &sn, &cs);
        if (head < s.nq) {
            const float a = pr[head * hd + i], bb = pr[head * hd + i + half];
            float* qo = s.qrot + (int64_t)row * qw + head * hd;
            qo[i] = a * cs - bb * sn;
            qo[i + half] = bb * cs + a * sn;
        } else {
            const int g = head - s.nq;
            const float* kp = pr + 2 * qw + g * hd;
            bf16_t* ko = kc + (((int64_t)b * s.nkv + g) * s.Lmax + P) * hd;
            ko[i] = f2bf(kp[i] * cs - kp[i + half] * sn);
            ko[i + half] = f2bf(kp[i + half] * cs + kp[i] * sn);
        }
    }
    if (head >= s.nq) {
        const int g = head - s.nq;
        const float* vp = pr + 2 * qw + s.nkv * hd + g * hd;
        bf16_t* vo = vc + (((int64_t)b * s.nkv + g) * s.Lmax + P) * hd;
        for (int d = lane; d < hd; d += 32) vo[d] = f2bf(vp[d]);
    }
}

// One attention partial: query head h of one row over one chunk of keys (the
// arithmetic of k_attn_partial's warps).  ex: this warp's 32 floats of scratch.
__device__ void sk_partial_item(const SkParams& s, int ia, int row, int h, int ch, int lane, float* ex) {
    const int b = row / s.T, t = row % s.T;
    const int P = s.pos[b] + t;
    if (P < 0 || P >= s.Lmax) return;
    const int key0 = ch * ATTN_CHUNK;
    if (key0 > P) return;
    const int nk = min(ATTN_CHUNK, P + 1 - key0);
    const int hd = s.hd, group = s.nq / s.nkv, g = h / group;
    const size_t kv_half = (size_t)s.B * s.nkv * s.Lmax * hd;
    const bf16_t* K = s.kv + (size_t)ia * 2 * kv_half + ((int64_t)b * s.nkv + g) * s.Lmax * hd;
    const bf16_t* V = K + kv_half;
    const float* q = s.qrot + (int64_t)row * s.nq * hd + (int64_t)h * hd;
    float sc = -INFINITY;
    if (lane < nk) {
        const bf16_t* kr = K + (int64_t)(key0 + lane) * hd;
        float d = 0.f;
        for (int e = 0; e < hd; e += 8) {
            const uint4 kv = *reinterpret_cast<const uint4*>(kr + e);
            const float4 q0 = *reinterpret_cast<const float4*>(q + e);
            const float4 q1 = *reinterpret_cast<const float4*>(q + e + 4);
            d = fmaf(q0.x, bf_lo(kv.x), d); d = fmaf(q0.y, bf_hi(kv.x), d);
            d = fmaf(q0.z, bf_lo(kv.y), d); d = fmaf(q0.w, bf_hi(kv.y), d);
            d = fmaf(q1.x, bf_lo(kv.z), d); d = fmaf(q1.y, bf_hi(kv.z), d);
            d = fmaf(q1.z, bf_lo(kv.w), d); d = fmaf(q1.w, bf_hi(kv.w), d);
        }
        sc = d * (1.0f / sqrtf((float)hd));
    }
    float m = sc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float e = (lane < nk) ? expf(sc - m) : 0.f;
    const float l = warp_sum(e);
    ex[lane] = e;
    __syncwarp();
    float* dst = s.part + (((int64_t)row * s.nq + h) * s.max_chunks + ch) * (hd + 2);
    for (int d0 = lane * 8; d0 < hd; d0 += 256) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < nk; ++j) {
            const uint4 vv = *reinterpret_cast<const uint4*>(V + (int64_t)(key0 + j) * hd + d0);
            const float wgt = ex[j];
            acc[0] = fmaf(wgt, bf_lo(vv.x), acc[0]); acc[1] = fmaf(wgt, bf_hi(vv.x), acc[1]);
            acc[2] = fmaf(wgt, bf_lo(vv.y), acc[2]); acc[3] = fmaf(wgt, bf_hi(vv.y), acc[3]);
            acc[4] = fmaf(wgt, bf_lo(vv.z), acc[4]); acc[5] = fmaf(wgt, bf_hi(vv.z), acc[5]);
            acc[6] = fmaf(wgt, bf_lo(vv.w), acc[6]); acc[7] = fmaf(wgt, bf_hi(vv.w), acc[7]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[2 + d0 + i] = acc[i];
    }
    if (lane == 0) { dst[0] = m; dst[1] = l; }
    __syncwarp();
}

// Merge the chunk partials of query head h of one row, times sigmoid(gate)
// (per dimension, the arithmetic of k_attn_merge).
__device__ void sk_merge_item(const SkParams& s, int row, int h, int lane) {
    const int b = row / s.T, t = row % s.T;
    const int P = s.pos[b] + t;
    const int hd = s.hd;
    bf16_t* out = s.attn + (int64_t)row * s.nq * hd + (int64_t)h * hd;
    if (P < 0 || P >= s.Lmax) {
        for (int d = lane; d < hd; d += 32) out[d] = 0;
        return;
    }
    const int nch = P / ATTN_CHUNK + 1;
    const float* base = s.part + ((int64_t)row * s.nq + h) * s.max_chunks * (hd + 2);
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, base[c * (hd + 2)]);
    for (int d = lane; d < hd; d += 32) {
        float L = 0.f, acc = 0.f;
        for (int c = 0; c < nch; ++c) {
            const float* pc = base + c * (hd + 2);
            const float wgt = expf(pc[0] - M);
            L = fmaf(wgt, pc[1], L);
            acc = fmaf(wgt, pc[2 + d], acc);
        }
        const float gate = s.proj[(int64_t)row * s.proj_ld + s.nq * hd + (int64_t)h * hd + d];
        out[d] = f2bf(acc / L * sigmoid_f(gate));
    }
}

// Argmax of each row over the CTAs' partials; positions advance by T.
__device__ void sk_final(const SkParams& s, int lane) {
    const int G = gridDim.x;
    for (int n = 0; n < s.M; ++n) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        bool nan = false;
        for (int g = lane; g < G; g += 32) {
            const int i = s.besti[n * G + g];
            const float v = s.bestv[n * G + g];
            if (i < 0) { nan = true; continue; }
            if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        nan = __any_sync(0xffffffffu, nan);
        if (lane == 0) {
            s.argmax[n] = nan ? -1 : bi;
            if (nan) set_status(s.status, HGD_ERR_NAN);
        }
    }
    if (lane == 0)
        for (int b = 0; b < s.B; ++b) s.pos[b] += s.T;
}

// ------------------------------------------------------------------ kernel

// Consumer side of one GEMV phase: prologue, this CTA's items, epilogue.
template <int PRO, int EPI>
__device__ void sk_gemv_phase(const SkParams& s, const GemvParams& p, uint8_t* ring, uint64_t* full,
                              uint64_t* empty, bf16_t* xs, float* cbuf, float* amax_v, int* amax_i,
                              int& wseq, volatile int* cta_abort, int warp, int lane, int phase) {
    const int seq_base = wseq;
    const int tid = threadIdx.x;
    if (!*cta_abort) gv_prologue<8, PRO>(p, xs, tid, warp, lane, nullptr);
    named_bar(1, SK_CW * 32);
    const int XS = p.K + GV_PAD;
    const int r8 = lane >> 2, c = lane & 3;
    const int steps_total = p.K >> 5;
    const int nsl = p.split ? 1 : p.nks;
    const int nmine = sk_cta_items(p.n_items);
    const bf16_t* xb = xs + r8 * XS + 8 * c;
    float* cb = cbuf + warp * GV_ROWS * 8;
    GvBest<1> best;
    best.init();
    for (int i = warp; i < nmine; i += SK_CW) {
        const int u = blockIdx.x + i * gridDim.x;
        const int rb = p.split ? u / p.nks : u;
        const int s0 = p.split ? u % p.nks : 0;
        float yacc[1][4];
        bool ok = !*cta_abort;
        for (int sl = 0; sl < nsl; ++sl) {
            const int seq = wseq++;  // this warp's slab sequence number
            const int slot = warp * SK_NSW + seq % SK_NSW;
            const uint32_t par = (uint32_t)((seq / SK_NSW) & 1);
            if (ok) {
                bool got = true;
                if (lane == 0) got = mbar_wait_bounded(&full[slot], par, cta_abort);
                got = __shfl_sync(0xffffffffu, got, 0);
                if (got) got = __all_sync(0xffffffffu, mbar_try_wait(&full[slot], par));
                if (!got) {
                    if (lane == 0) {
                        if (!*cta_abort && atomicCAS(&s.bar[4], 0u, 2u) == 0u) {
                            const volatile int* pr = reinterpret_cast<const volatile int*>(cta_abort) + 1;
                            s.bar[5] = (unsigned)phase;
                            s.bar[6] = blockIdx.x;
                            s.bar[7] = (unsigned)seq;
                            s.bar[8] = (unsigned)pr[0];
                            s.bar[9] = (unsigned)pr[1];
                            s.bar[10] = (unsigned)warp;
                            s.bar[12] = (unsigned)seq_base;
                            unsigned fb = 0, eb = 0;
                            for (int q = 0; q < SK_NSLOT; ++q) {
                                fb |= (mbar_try_wait(&full[q], 0) ? 1u : 0u) << (2 * q);
                                fb |= (mbar_try_wait(&full[q], 1) ? 2u : 0u) << (2 * q);
                                eb |= (mbar_try_wait(&empty[q], 0) ? 1u : 0u) << (2 * q);
                                eb |= (mbar_try_wait(&empty[q], 1) ? 2u : 0u) << (2 * q);
                            }
                            s.bar[11] = fb;
                            s.bar[13] = eb;
                        }
                        sk_timeout(s.bar, s.status, 2u, (unsigned)phase, (unsigned)seq);
                        *cta_abort = 1;
                    }
                    ok = false;
                }
            }
            const int sg = s0 + sl;  // slab index within the row block
            const int nstep = min(GV_SLAB_STEPS, steps_total - sg * GV_SLAB_STEPS);
            float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok) {
                const bf16_t* tile = reinterpret_cast<const bf16_t*>(ring + slot * SK_SLAB_BYTES);
#pragma unroll
                for (int jj = 0; jj < GV_SLAB_STEPS; ++jj) {
                    if (jj < nstep) {
                        const uint4 a0 = lds128(tile + jj * 512 + lane * 8);
                        const uint4 a1 = lds128(tile + jj * 512 + 256 + lane * 8);
                        const uint4 Bv = lds128(xb + (sg * GV_SLAB_STEPS + jj) * 32);
                        float (&acc)[4] = (jj & 1) ? c1 : c0;
                        mma_bf16_16816(acc, a0.x, a1.x, a0.y, a1.y, Bv.x, Bv.y);
                        mma_bf16_16816(acc, a0.z, a1.z, a0.w, a1.w, Bv.z, Bv.w);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[slot]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float part = c0[q] + c1[q];
                yacc[0][q] = (p.split || sl == 0) ? part : yacc[0][q] + part;
            }
        }
        if (ok) gv_finish<1, EPI>(p, rb, s0, yacc, lane, cb, best);
    }
    if (EPI == EPI_ARGMAX)
        gv_argmax_cta<1>(p, best, amax_v, amax_i, warp, lane, tid, SK_CW, blockIdx.x, gridDim.x, true);
}

template <int KPL>
__global__ void __launch_bounds__(SK_THREADS, 1) k_stack(const __grid_constant__ SkParams s) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t* ring = smem;
    bf16_t* xs = reinterpret_cast<bf16_t*>(smem + SK_NSLOT * SK_SLAB_BYTES);
    float* cbuf = reinterpret_cast<float*>(smem + SK_NSLOT * SK_SLAB_BYTES + s.x_bytes);  // [CW][16][8]
    float* amax_v = cbuf + SK_CW * GV_ROWS * 8;
    int* amax_i = reinterpret_cast<int*>(amax_v + SK_CW * 8);
    float* exbuf = reinterpret_cast<float*>(amax_i + SK_CW * 8);  // [CW][32]
    uint64_t* full = reinterpret_cast<uint64_t*>(exbuf + SK_CW * 32);
    uint64_t* empty = full + SK_NSLOT;
    volatile int* cta_abort = reinterpret_cast<volatile int*>(empty + SK_NSLOT);
    volatile int* prod = cta_abort + 1;  // [0] producer's next sequence number, [1] 1 while it waits

    if (tid == 0) {
        for (int i = 0; i < SK_NSLOT; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        *cta_abort = 0;
        prod[0] = 0;
        prod[1] = 0;
        mbar_fence_init();
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer
    if (warp == SK_CW) {
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        int wseq[SK_CW];
        for (int w = 0; w < SK_CW; ++w) wseq[w] = 0;
        int pid = -1;
        bool ok = true;
        for (int l = 0; l <= s.L && ok; ++l) {
            const int nph = (l == s.L) ? 1 : sk_nphase(s, l);
            for (int j = 0; j < nph && ok; ++j) {
                ++pid;
                const int kind = sk_kind(s, l, j);
                if (!sk_is_gemv(kind)) continue;
                GemvParams p;
                sk_gemv_params(s, kind, l, 0, p);
                const int steps_total = p.K >> 5;
                const int nsl = p.split ? 1 : p.nks;
                const int nmine = sk_cta_items(p.n_items);
                // warp w owns items w, w + CW, ...; its k-th slab of the phase is slab
                // k % nsl of its (k / nsl)-th item.  Feed the warps one slab each in turn.
                const int per_warp_max = ((nmine + SK_CW - 1) / SK_CW) * nsl;
                for (int k = 0; k < per_warp_max && ok; ++k) {
                    for (int w = 0; w < SK_CW && ok; ++w) {
                        const int i = w + (k / nsl) * SK_CW;
                        if (i >= nmine) continue;
                        const int sl = k % nsl;
                        const int u = blockIdx.x + i * gridDim.x;
                        const int rb = p.split ? u / p.nks : u;
                        const int s0 = p.split ? u % p.nks : 0;
                        const int q = wseq[w]++;
                        const int slot = w * SK_NSW + q % SK_NSW;
                        const uint32_t par = (uint32_t)((q / SK_NSW) & 1);
                        prod[0] = q;
                        prod[1] = 1;
                        const bool free_slot = mbar_wait_bounded(&empty[slot], par ^ 1, cta_abort);
                        prod[1] = 0;
                        if (!free_slot || ld_acquire_u32(&s.bar[2])) {
                            if (!ld_acquire_u32(&s.bar[2])) sk_timeout(s.bar, s.status, 3u, (unsigned)pid, (unsigned)q);
                            wseq[w]--;
                            ok = false;
                            break;
                        }
                        const int sg = s0 + sl;
                        const int nstep = min(GV_SLAB_STEPS, steps_total - sg * GV_SLAB_STEPS);
                        const uint32_t bytes = (uint32_t)nstep * 1024u;
                        mbar_arrive_expect_tx(&full[slot], bytes);
                        bulk_g2s(ring + slot * SK_SLAB_BYTES,
                                 p.W + gv_tile_elem(rb, sg * GV_SLAB_STEPS, steps_total, 0, 0), bytes, &full[slot],
                                 pol);
                    }
                }
            }
        }
        // Do not leave while a copy into this CTA's shared memory is in flight.
        for (int w = 0; w < SK_CW; ++w)
            for (int q = max(0, wseq[w] - SK_NSW); q < wseq[w]; ++q)
                (void)mbar_wait_bounded(&full[w * SK_NSW + q % SK_NSW], (uint32_t)((q / SK_NSW) & 1), nullptr);
        return;
    }

    // --------------------------------------------------------------- consumers
    int wseq = 0;  // this warp's slab sequence number across all phases
    int ig = 0, ia = 0, pid = -1;
    bool first = true;
    for (int l = 0; l <= s.L; ++l) {
        const bool att = l < s.L && sk_attn(s, l);
        const int nph = (l == s.L) ? 2 : sk_nphase(s, l);
        for (int j = 0; j < nph; ++j) {
            const int kind = sk_kind(s, l, j);
            ++pid;
            if (!first) sk_grid_sync(s, cta_abort, pid);
            first = false;
            if (s.trace && blockIdx.x == 0 && threadIdx.x == 0 && pid < 256) s.trace[pid] = globaltimer();
            const bool live = !*cta_abort;
            if (sk_is_gemv(kind)) {
                GemvParams p;
                sk_gemv_params(s, kind, l, ig, p);
                switch (kind) {
                    case SK_IN_GDN:
                        if (l == 0) sk_gemv_phase<PRO_EMBED_RMSNORM, EPI_QKV_CONV>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        else sk_gemv_phase<PRO_RMSNORM, EPI_QKV_CONV>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                    case SK_IN_ATT:
                        if (l == 0) sk_gemv_phase<PRO_EMBED_RMSNORM, EPI_F32>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        else sk_gemv_phase<PRO_RMSNORM, EPI_F32>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                    case SK_OUT_GDN:
                        sk_gemv_phase<PRO_GATED_NORM, EPI_RESID>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                    case SK_OUT_ATT: case SK_DOWN:
                        sk_gemv_phase<PRO_COPY, EPI_RESID>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                    case SK_SWIGLU:
                        sk_gemv_phase<PRO_RMSNORM, EPI_SWIGLU>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                    default:
                        sk_gemv_phase<PRO_RMSNORM, EPI_ARGMAX>(s, p, ring, full, empty, xs, cbuf, amax_v, amax_i, wseq, cta_abort, warp, lane, pid);
                        break;
                }
                continue;
            }
            // the phases without weights: items spread over the warps of all CTAs
            const int gw = warp * gridDim.x + blockIdx.x, nw = gridDim.x * SK_CW;
            if (kind == SK_GDN) {
                const int rg = s.dv / GDN_RPW;
                const int n = s.B * s.H * rg;
                for (int it = gw; live && it < n; it += nw) {
                    const int b = it / (s.H * rg), h = (it / rg) % s.H, r = it % rg;
                    sk_gdn_item<KPL>(s, l, ig, b, h, r * GDN_RPW, lane);
                }
            } else if (kind == SK_ROPE) {
                const int nh = s.nq + s.nkv, n = s.M * nh;
                for (int it = gw; live && it < n; it += nw) sk_rope_item(s, ia, it / nh, it % nh, lane);
            } else if (kind == SK_PART) {
                const int n = s.M * s.nq * s.max_chunks;
                for (int it = gw; live && it < n; it += nw) {
                    const int row = it / (s.nq * s.max_chunks), h = (it / s.max_chunks) % s.nq;
                    sk_partial_item(s, ia, row, h, it % s.max_chunks, lane, exbuf + warp * 32);
                }
            } else if (kind == SK_MERGE) {
                const int n = s.M * s.nq;
                for (int it = gw; live && it < n; it += nw) sk_merge_item(s, it / s.nq, it % s.nq, lane);
            } else if (kind == SK_FINAL) {
                if (live && blockIdx.x == 0 && warp == 0) sk_final(s, lane);
            }
        }
        if (l < s.L) (att ? ia : ig)++;
    }
    if (s.trace && blockIdx.x == 0 && threadIdx.x == 0) s.trace[255] = globaltimer();
}

}  // namespace hgd
