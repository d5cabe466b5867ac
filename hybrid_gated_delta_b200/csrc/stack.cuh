// stack.cuh -- one cooperative launch for a whole decode step of the stack.
//
// "luce-megakernel HANDOFF.md", Architecture: all 24 layers of the decode step
// in one persistent kernel with synchronisation between layers (and its Known
// Issues: a grid-wide wait deadlocks unless every block is resident, hence a
// cooperative launch).  Built for B200 here, as a dataflow of phases:
//  * one CTA per SM: a producer warp and eight consumer warps;
//  * weights never depend on activations, so the producer walks the CTA's share
//    of every projection of the step in order and streams each 16-row x
//    256-column weight slab (8 KB, contiguous thanks to the fragment-ordered
//    packing) with one bulk copy (cp.async.bulk into this CTA's own shared memory, L2 evict-first)
//    into a CTA-wide ring of NS slots, across phase boundaries: HBM stays busy
//    while the consumers wait for the previous phase.  Slab g of the CTA's
//    sequence sits in slot g % NS and is consumed by warp g % 8 (NS is a
//    multiple of 8), so each slot is only ever waited on by one warp, strictly
//    in order, and an mbarrier phase parity never aliases;
//  * per layer five phases -- GDN: in-projection with the fused causal conv,
//    gated delta rule, out-projection with the gated RMSNorm, SwiGLU, down;
//    attention: in-projection with the fused RoPE and KV append, attention
//    partials, out-projection with the fused merge, SwiGLU, down -- then the LM
//    head with the argmax and the final argmax reduction;
//  * phases synchronise through monotonic counters, one per phase: each CTA
//    adds 1 (red.release) once its writes of phase p are done, and phase p + 1
//    starts when the counter of phase p reaches the grid size (ld.acquire);
//  * a work item is a whole 16-row block (its slabs spread over the warps, the
//    partials gathered in shared memory and added in slab order by the item's
//    warp), so each projection's epilogue -- residual add included -- runs
//    where the row is finished and the next phase reads only the residual
//    rows.  Items go to CTA (phase rotation + item) % grid, so phases with
//    fewer row blocks than CTAs land on different SMs from layer to layer and
//    the weight stream stays spread over all of them;
//  * every output has the arithmetic of the kernel chain (the same device
//    functions, the same slab order), so the two agree bit for bit;
//  * every wait is bounded; a wait that runs out sets HGD_ERR_TIMEOUT and a
//    global abort word, after which every CTA skips the remaining work.
#pragma once

#include "attn.cuh"
#include "gdn.cuh"
#include "gemv.cuh"

namespace hgd {

constexpr int SK_CW = 8;                        // consumer warps
constexpr int SK_CT = SK_CW * 32;               // consumer threads
constexpr int SK_THREADS = SK_CT + 32;          // + the producer warp
constexpr int SK_SLAB_BYTES = GV_SLAB_STEPS * 1024;
constexpr int SK_PB_SLAB = GV_ROWS * 8;         // floats of one slab partial in the partial buffer
constexpr int SK_MAXM = 8;                      // token rows per call (one MMA n-tile)
constexpr int SK_PHASES_PER_LAYER = 5;
constexpr int SK_MAX_PHASES = SK_PHASES_PER_LAYER * HGD_MAX_LAYERS + 2;
// control words: [0] abort, [1] what ran out first (1 phase counter, 2 weight
// slab, 3 free ring slot), [2] its phase, [3] its CTA, [4] its sequence number;
// then the attention merge counters [M][nq] (SK_MCNT_WORDS); the counter of
// phase p is word SK_CTRL_WORDS + SK_MCNT_WORDS + p * SK_CTR_STRIDE (own 128 B)
constexpr int SK_CTRL_WORDS = 32;
constexpr int SK_MCNT_WORDS = 1024;
constexpr int SK_CTR_STRIDE = 32;
constexpr int SK_TRACE_SLOTS = 512;             // phase start times of CTA 0; the end in the last
constexpr int SK_TRACE_CTAS = 256;              // CTAs the per-CTA phase times cover
constexpr int SK_TRACE_SLABS = 4096;            // slabs of CTA 0 the slab times cover

enum SkKind { SK_IN_GDN = 0, SK_GDN, SK_OUT_GDN, SK_IN_ATT, SK_PART, SK_OUT_ATT, SK_SWIGLU, SK_DOWN, SK_HEAD,
              SK_FINAL };

struct SkLayer { const bf16_t* w[HGD_W_LAYER_COUNT]; };

struct SkParams {
    int L, D, V, H, dk, dv, nq, nkv, hd, I, every;
    int Hk;            // GDN query/key heads; H (the value heads) is a multiple
    const bf16_t* head;  // the LM head [V][D] (packed): the embedding when tied
    int C, gdn_out, attn_out, proj_ld, kmax;
    float eps;
    double rope_inv1;  // base^(-2/hd)
    int B, T, M, Lmax, max_chunks;
    int ns, pb;      // ring slots (a multiple of SK_CW), slab partials the partial buffer holds
    const bf16_t* embed; const bf16_t* final_norm;
    float* S; float* conv; bf16_t* kv; int32_t* pos;
    bf16_t* resid;   // [M][D] residual rows (updated in place by the out- and down-projections)
    float* proj; float* obuf; float* qrot; float* part; bf16_t* mlp;
    bf16_t* attn;    // [M][nq*hd] merged attention output
    unsigned* mcnt;  // [M][nq] chunks finished per (row, head), zero between layers
    float* bestv; int32_t* besti;
    const int32_t* tokens; float* logits; int32_t* argmax; float* S_rec; float* tail_rec;
    int32_t* status;
    unsigned* bar;               // control words and phase counters (zeroed before the launch)
    unsigned long long* trace;   // [SK_TRACE_SLOTS] %globaltimer, or null
    unsigned long long* tdetail; // [SK_MAX_PHASES][SK_TRACE_CTAS][8] per-CTA phase times, or null
    unsigned long long* tslab;   // CTA 0: [SK_TRACE_SLABS][4] slab issue / ready / release / wait-start times, or null
    unsigned long long wait_ns;  // limit of each phase wait (kWaitLimitNs in normal calls)
    int dbg_skip_cta, dbg_skip_phase;  // diagnostic: this CTA leaves out its arrival at this phase (-1: none)
    SkLayer layer[HGD_MAX_LAYERS];
};

__device__ __forceinline__ bool sk_attn(const SkParams& s, int l) { return l % s.every == s.every - 1; }
__device__ __forceinline__ int sk_kind(const SkParams& s, int l, int j) {
    if (l == s.L) return j == 0 ? SK_HEAD : SK_FINAL;
    static constexpr int gdn[5] = {SK_IN_GDN, SK_GDN, SK_OUT_GDN, SK_SWIGLU, SK_DOWN};
    static constexpr int att[5] = {SK_IN_ATT, SK_PART, SK_OUT_ATT, SK_SWIGLU, SK_DOWN};
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
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned* sk_ctr(const SkParams& s, int p) {
    return s.bar + SK_CTRL_WORDS + SK_MCNT_WORDS + p * SK_CTR_STRIDE;
}

// Record the first wait that ran out; set the status and the abort word.
__device__ __forceinline__ void sk_timeout_w(unsigned* bar, int32_t* status, unsigned what, unsigned phase,
                                             unsigned seq) {
    if (atomicCAS(&bar[1], 0u, what) == 0u) {
        bar[2] = phase;
        bar[3] = blockIdx.x;
        bar[4] = seq;
    }
    set_status(status, HGD_ERR_TIMEOUT);
    atomicExch(&bar[0], 1u);
}
__device__ __forceinline__ void sk_timeout(const SkParams& s, unsigned what, unsigned phase, unsigned seq) {
    sk_timeout_w(s.bar, s.status, what, phase, seq);
}

// End of phase p in this CTA: once every consumer warp's writes are done (the
// CTA barrier orders them before thread 0's release), one release-add to the
// phase's counter.
__device__ __forceinline__ void sk_arrive(const SkParams& s, int p) {
    named_bar(1, SK_CT);
    if (threadIdx.x == 0 && !((int)blockIdx.x == s.dbg_skip_cta && p == s.dbg_skip_phase))
        red_release_add(sk_ctr(s, p), 1u);
}

// Named barrier over the consumer threads that also ANDs a predicate: every
// thread gets the same answer, so branches around later barriers stay uniform.
__device__ __forceinline__ bool sk_bar_and(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(SK_CT)
        : "memory");
    return r != 0;
}

// Wait until every CTA has arrived at the end of phase p.  Lane 0 of warps
// 0..SK_POLLERS-1 poll the counter (one poller: fewer loads on the counter's
// line measured faster than four staggered ones); the first to see it raises
// `seen` (shared) for the others; the consumer warps then meet at a named
// barrier.  False, in every consumer thread, on an abort or a timeout.
constexpr int SK_POLLERS = 1;
__device__ bool sk_wait(const SkParams& s, volatile int* cta_abort, volatile int* seen, int p) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0 && warp < SK_POLLERS && !*cta_abort) {
        const unsigned* c = sk_ctr(s, p);
        const unsigned target = gridDim.x;
        if (warp) __nanosleep(120u * (unsigned)warp);
        if (*seen != p && ld_acquire_u32(c) < target) {
            const unsigned long long t0 = globaltimer();
            unsigned it = 0;
            while (*seen != p && ld_acquire_u32(c) < target) {
                if ((++it & 31u) == 0u) {
                    if (ld_acquire_u32(&s.bar[0])) { *cta_abort = 1; break; }
                    if (globaltimer() - t0 > s.wait_ns) {
                        // whichever poller runs out first records it (the record is
                        // first-wins); the others then leave through `seen`
                        sk_timeout(s, 1u, (unsigned)p, 0u);
                        *cta_abort = 1;
                        break;
                    }
                }
            }
        }
        *seen = p;
    }
    return sk_bar_and(!*cta_abort);
}

// GEMV parameters of a phase (the same fields the kernel chain's launch uses).
__device__ __forceinline__ void sk_gemv_params(const SkParams& s, int kind, int l, int ig, int ia, GemvParams& p) {
    p = GemvParams{};
    const bf16_t* const* w = l < s.L ? s.layer[l].w : nullptr;
    p.packed = 1;
    p.M = s.M;
    p.eps = s.eps;
    p.status = s.status;
    bool swi = false;
    switch (kind) {
        case SK_IN_GDN: {
            const size_t c_layer = (size_t)s.B * (GV_CONV_K - 1) * s.C;
            const size_t trec_layer = (size_t)s.B * s.T * (GV_CONV_K - 1) * s.C;
            p.W = w[HGD_W_IN]; p.N = s.gdn_out; p.K = s.D; p.norm_w = w[HGD_W_IN_NORM];
            p.y = s.proj; p.y_ld = s.proj_ld;
            p.conv_w = w[HGD_W_CONV]; p.conv_tail = s.conv + ig * c_layer;
            p.conv_rec = s.tail_rec ? s.tail_rec + ig * trec_layer : nullptr;
            p.conv_C = s.C; p.conv_T = s.T; p.m0 = 0;
            break;
        }
        case SK_IN_ATT: {
            const size_t kv_half = (size_t)s.B * s.nkv * s.Lmax * s.hd;
            p.W = w[HGD_W_IN]; p.N = s.attn_out; p.K = s.D; p.norm_w = w[HGD_W_IN_NORM];
            p.y = s.proj; p.y_ld = s.proj_ld;
            p.rope_nq = s.nq; p.rope_nkv = s.nkv; p.rope_hd = s.hd; p.rope_Lmax = s.Lmax; p.rope_inv1 = s.rope_inv1;
            p.rope_q = s.qrot; p.rope_k = s.kv + (size_t)ia * 2 * kv_half; p.rope_v = p.rope_k + kv_half;
            p.rope_pos = s.pos; p.conv_T = s.T; p.m0 = 0;
            break;
        }
        case SK_OUT_GDN:
            p.W = w[HGD_W_OUT]; p.N = s.D; p.K = s.H * s.dv;
            p.gnorm_w = w[HGD_W_GNORM]; p.gn_d = s.dv;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        case SK_OUT_ATT:
            p.W = w[HGD_W_OUT]; p.N = s.D; p.K = s.nq * s.hd;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        case SK_SWIGLU:
            p.W = w[HGD_W_GATE]; p.N = s.I; p.K = s.D; swi = true; p.norm_w = w[HGD_W_POST_NORM];
            p.y = s.mlp; p.y_ld = s.I;
            break;
        case SK_DOWN:
            p.W = w[HGD_W_DOWN]; p.N = s.D; p.K = s.I;
            p.y = s.resid; p.y_ld = s.D; p.resid = s.resid; p.resid_ld = s.D;
            break;
        default:  // SK_HEAD
            p.W = s.head; p.N = s.V; p.K = s.D; p.norm_w = s.final_norm;
            p.logits = s.logits; p.logits_ld = s.V; p.best_v = s.bestv; p.best_i = s.besti;
            break;
    }
    p.nks = gv_slabs(p.K);
    p.n_rowblk = swi ? (p.N + 7) / 8 : (p.N + GV_ROWS - 1) / GV_ROWS;
    p.split = 0;
    p.n_items = p.n_rowblk;
}

// The norm gains the prologue of phase `kind` of layer l reads (the RMSNorm
// before the in-projections, the SwiGLU and the LM head; the gated norm before
// the GDN out-projection), or null; n: their count.
__device__ __forceinline__ const bf16_t* sk_gains(const SkParams& s, int kind, int l, int& n) {
    n = s.D;
    switch (kind) {
        case SK_IN_GDN: case SK_IN_ATT: return s.layer[l].w[HGD_W_IN_NORM];
        case SK_SWIGLU: return s.layer[l].w[HGD_W_POST_NORM];
        case SK_HEAD: return s.final_norm;
        case SK_OUT_GDN: n = s.dv; return s.layer[l].w[HGD_W_GNORM];
        default: n = 0; return nullptr;
    }
}


// This CTA's place in phase `pid`'s item order (a rotation that moves from
// phase to phase), and its items c, c + G, c + 2G, ... of n.
__device__ __forceinline__ int sk_vcta(int pid) {
    const int G = gridDim.x;
    return (int)((blockIdx.x + (unsigned)pid * 37u) % (unsigned)G);
}
__device__ __forceinline__ int sk_cta_items(int n, int c) {
    const int G = gridDim.x;
    return c < n ? (n - c + G - 1) / G : 0;
}

// ------------------------------------------------------------------ prologues
// xs rows hold the M token rows of the phase's GEMV input (bf16, row stride
// K + GV_PAD); only rows < M exist.

// The residual rows (bf16) into xs.
__device__ void sk_pro_resid(const SkParams& s, bf16_t* xs) {
    const int K = s.D, XS = K + GV_PAD, cpr = K / 8;
    for (int e = threadIdx.x; e < s.M * cpr; e += SK_CT) {
        const int m = e / cpr, c = e % cpr;
        *reinterpret_cast<uint4*>(xs + m * XS + c * 8) =
            *reinterpret_cast<const uint4*>(s.resid + (int64_t)m * K + c * 8);
    }
}

// RMSNorm of the residual rows in xs, in place, one warp per row, with gains gb
// (shared): the arithmetic of gv_prologue's RMSNorm.
__device__ void sk_pro_rmsnorm(const SkParams& s, bf16_t* xs, const bf16_t* gb, int warp, int lane) {
    const int K = s.D, XS = K + GV_PAD;
    for (int m = warp; m < s.M; m += SK_CW) {
        bf16_t* row = xs + m * XS;
        float ss = 0.f;
        for (int c = lane; c < K / 8; c += 32) {
            const uint4 v = lds128(row + c * 8);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float a = bf_lo(w4[q]), b = bf_hi(w4[q]);
                ss = fmaf(a, a, ss);
                ss = fmaf(b, b, ss);
            }
        }
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)K + s.eps);
        for (int c = lane; c < K / 8; c += 32) {
            const uint4 v = lds128(row + c * 8);
            const uint4 g = lds128(gb + c * 8);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            const uint32_t g4[4] = {g.x, g.y, g.z, g.w};
            uint32_t o4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                o4[q] = pack_bf2(bf_lo(w4[q]) * r * bf_lo(g4[q]), bf_hi(w4[q]) * r * bf_hi(g4[q]));
            *reinterpret_cast<uint4*>(row + c * 8) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
    }
}

// RMSNorm of the residual rows straight from global memory into xs, with gains
// gb (shared; this thread's copies of them waited for here): the arithmetic of
// gv_prologue's RMSNorm.  Every warp loads its lanes' chunks (chunk c = lane +
// 32 j) of a row and forms the same sum of squares in the same order, so every
// warp holds the same scale; the lanes l with l % 8 == warp write their chunks.
// Needs D % 256 == 0 and D <= 1024.
constexpr int SK_NORM_MAXJ = 4;
__device__ void sk_pro_resid_rmsnorm(const SkParams& s, bf16_t* xs, const bf16_t* gb, int warp, int lane) {
    const int K = s.D, XS = K + GV_PAD, nj = K / 256;
    uint4 v[SK_NORM_MAXJ][1];
    for (int m = 0; m < s.M; ++m) {
        const bf16_t* src = s.resid + (int64_t)m * K;
#pragma unroll
        for (int j = 0; j < SK_NORM_MAXJ; ++j)
            if (j < nj) v[j][0] = *reinterpret_cast<const uint4*>(src + (lane + 32 * j) * 8);
        if (m == 0) {
            cp_async_wait_prior();
            named_bar(1, SK_CT);
        }
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < SK_NORM_MAXJ; ++j)
            if (j < nj) {
                const uint32_t w4[4] = {v[j][0].x, v[j][0].y, v[j][0].z, v[j][0].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a = bf_lo(w4[q]), b = bf_hi(w4[q]);
                    ss = fmaf(a, a, ss);
                    ss = fmaf(b, b, ss);
                }
            }
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)K + s.eps);
        if ((lane & (SK_CW - 1)) == warp) {
            bf16_t* row = xs + m * XS;
#pragma unroll
            for (int j = 0; j < SK_NORM_MAXJ; ++j)
                if (j < nj) {
                    const int c = lane + 32 * j;
                    const uint4 g = lds128(gb + c * 8);
                    const uint32_t w4[4] = {v[j][0].x, v[j][0].y, v[j][0].z, v[j][0].w};
                    const uint32_t g4[4] = {g.x, g.y, g.z, g.w};
                    uint32_t o4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        o4[q] = pack_bf2(bf_lo(w4[q]) * r * bf_lo(g4[q]), bf_hi(w4[q]) * r * bf_hi(g4[q]));
                    *reinterpret_cast<uint4*>(row + c * 8) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
        }
    }
}

// Layer 0: the embedding rows of the tokens (the packed embedding, gathered by
// 16-byte chunks) into xs, CTA 0 writes them to the residual; a token outside
// the vocabulary gives a zero row and HGD_ERR_INVALID_ARG.
__device__ void sk_pro_embed(const SkParams& s, bf16_t* xs) {
    const int K = s.D, XS = K + GV_PAD, cpr = K / 8;
    for (int e = threadIdx.x; e < s.M * cpr; e += SK_CT) {
        const int m = e / cpr, c = e % cpr;
        const int tok = s.tokens[m];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (tok < 0 || tok >= s.V) {
            if (c == 0) set_status(s.status, HGD_ERR_INVALID_ARG);
        } else {
            v = *reinterpret_cast<const uint4*>(s.embed + gv_packed_chunk(tok, c, K >> 5));
        }
        *reinterpret_cast<uint4*>(xs + m * XS + c * 8) = v;
        if (blockIdx.x == 0) *reinterpret_cast<uint4*>(s.resid + (int64_t)m * K + c * 8) = v;
    }
}

// GDN out-projection input: per token row and head of width dv, the gated
// RMSNorm o * rsqrt(mean(o^2) + eps) * w * silu(bf16(z)) (gv_prologue's), gains
// gb in shared memory.  A warp takes its (row, head) pairs two at a time with
// every load of both issued first (dv <= 128); wider heads loop.
__device__ void sk_pro_gated(const SkParams& s, const GemvParams& p, const bf16_t* gb, bf16_t* xs, int warp,
                             int lane) {
    const int K = p.K, XS = K + GV_PAD, d = s.dv, nh = K / d, n = s.M * nh;
    if (d <= 128) {
        const int nk = d / 32;
        for (int e0 = warp; e0 < n; e0 += 2 * SK_CW) {
            float o[2][4], z[2][4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * SK_CW;
                const int m = e / nh, h = e % nh;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    o[u][k] = 0.f;
                    z[u][k] = 0.f;
                    if (e < n && k < nk) {
                        o[u][k] = s.obuf[(int64_t)m * K + h * d + lane + 32 * k];
                        z[u][k] = s.proj[(int64_t)m * s.proj_ld + s.C + h * d + lane + 32 * k];
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int e = e0 + u * SK_CW;
                if (e >= n) break;
                const int m = e / nh, h = e % nh;
                float ss = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < nk) ss = fmaf(o[u][k], o[u][k], ss);
                ss = warp_sum(ss);
                const float r = rsqrtf(ss / (float)d + s.eps);
                bf16_t* dst = xs + m * XS + h * d;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (k < nk) {
                        const int i = lane + 32 * k;
                        const float zb = bf2f(f2bf(z[u][k]));
                        dst[i] = f2bf(o[u][k] * r * bf2f(gb[i]) * silu_f(zb));
                    }
            }
        }
        return;
    }
    for (int e = warp; e < n; e += SK_CW) {
        const int m = e / nh, h = e % nh;
        bf16_t* dst = xs + m * XS + h * d;
        const float* orow = s.obuf + (int64_t)m * K + h * d;
        const float* zrow = s.proj + (int64_t)m * s.proj_ld + s.C + h * d;
        float ss = 0.f;
        for (int i = lane; i < d; i += 32) ss = fmaf(orow[i], orow[i], ss);
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)d + s.eps);
        for (int i = lane; i < d; i += 32) {
            const float zb = bf2f(f2bf(zrow[i]));
            dst[i] = f2bf(orow[i] * r * bf2f(gb[i]) * silu_f(zb));
        }
    }
}

// Merge of the chunk partials of (row, query head h) -> out [hd] bf16, times
// sigmoid(gate), by one warp.  Per dim d the arithmetic of attn_merge_dim:
// M = max_c m_c, then in chunk order w_c = exp(m_c - M), L += w_c l_c,
// acc_d += w_c acc_c[d].  Lane c % 32 loads chunk c's (m, l) and computes w_c
// (shared by shuffles); lane j holds the hd / 32 contiguous dims from
// j * hd / 32 (hd one of 32, 64, 128, 256) and loads them for SK_MB chunks at
// a time.
constexpr int SK_MB = 8;
template <int DPL>
__device__ void sk_merge_head_t(const float* base, int nch, const float* gate, bf16_t* out, int lane) {
    constexpr int hd = 32 * DPL, NV = (DPL + 3) / 4;  // float4s per lane per chunk
    const int d0 = lane * DPL;
    float L = 0.f, acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    float Mx = -INFINITY;
    for (int c = lane; c < nch; c += 32) Mx = fmaxf(Mx, __ldcg(base + (int64_t)c * (hd + 2)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Mx = fmaxf(Mx, __shfl_xor_sync(0xffffffffu, Mx, o));
    for (int cb = 0; cb < nch; cb += 32) {
        const int c = cb + lane;
        float wl = 0.f, ll = 0.f;
        if (c < nch) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(base + (int64_t)c * (hd + 2)));
            wl = expf(ml.x - Mx);
            ll = ml.y;
        }
        const int nb = min(32, nch - cb);
        for (int j0 = 0; j0 < nb; j0 += SK_MB) {
            float v[SK_MB][DPL];
#pragma unroll
            for (int u = 0; u < SK_MB; ++u) {
                const float* pc = base + (int64_t)(cb + j0 + u) * (hd + 2) + 2 + d0;
                if (j0 + u < nb) {
                    if (DPL >= 4) {
#pragma unroll
                        for (int k = 0; k < NV; ++k) {
                            const float2 a = __ldcg(reinterpret_cast<const float2*>(pc + 4 * k));
                            const float2 b = __ldcg(reinterpret_cast<const float2*>(pc + 4 * k + 2));
                            v[u][4 * k] = a.x; v[u][4 * k + 1] = a.y; v[u][4 * k + 2] = b.x; v[u][4 * k + 3] = b.y;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < DPL; ++i) v[u][i] = __ldcg(pc + i);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < DPL; ++i) v[u][i] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < SK_MB; ++u) {
                const float w = __shfl_sync(0xffffffffu, wl, (j0 + u) & 31);
                const float lc = __shfl_sync(0xffffffffu, ll, (j0 + u) & 31);
                if (j0 + u < nb) {
                    L = fmaf(w, lc, L);
#pragma unroll
                    for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, v[u][i], acc[i]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) out[d0 + i] = f2bf(acc[i] / L * sigmoid_f(gate[d0 + i]));
}

// Down-projection input: the SwiGLU rows (bf16) as they are.
__device__ void sk_pro_copy(const SkParams& s, const bf16_t* x, int K, bf16_t* xs) {
    const int XS = K + GV_PAD, cpr = K / 8;
    for (int e = threadIdx.x; e < s.M * cpr; e += SK_CT) {
        const int m = e / cpr, c = e % cpr;
        *reinterpret_cast<uint4*>(xs + m * XS + c * 8) = *reinterpret_cast<const uint4*>(x + (int64_t)m * K + c * 8);
    }
}

// ------------------------------------------------------------ GEMV consumer
struct SkRing {
    uint8_t* ring;
    uint64_t* full;
    uint64_t* empty;
    int ns;
};

// Wait for the weight slab of CTA sequence number g (slot g % ns); false if the
// wait ran out or the CTA aborted.  Every lane observes the completed phase.
__device__ __forceinline__ bool sk_slab_wait(unsigned* bar, int32_t* status, unsigned long long* tslab,
                                             const SkRing& r, int g, volatile int* cta_abort, int phase, int lane) {
    const int slot = g % r.ns;
    const uint32_t par = (uint32_t)((g / r.ns) & 1);
    if (tslab && blockIdx.x == 0 && lane == 0 && g < SK_TRACE_SLABS) tslab[g * 4 + 3] = globaltimer();
    bool got = true;
    if (lane == 0) got = mbar_wait_bounded(&r.full[slot], par, cta_abort);
    got = __shfl_sync(0xffffffffu, got, 0);
    if (got) got = __all_sync(0xffffffffu, mbar_try_wait(&r.full[slot], par));
    if (!got && lane == 0 && !*cta_abort) {
        sk_timeout_w(bar, status, 2u, (unsigned)phase, (unsigned)g);
        *cta_abort = 1;
    }
    if (tslab && blockIdx.x == 0 && lane == 0 && g < SK_TRACE_SLABS) tslab[g * 4 + 1] = globaltimer();
    return got;
}

// 16 x 8 partial of one slab: chain 0 (even steps) + chain 1 (odd steps), the
// per-slab arithmetic of k_gemv.  A full slab (every slab of a K that is a
// multiple of 256) takes a loop without per-step guards, which lets every
// shared-memory load of the slab issue ahead of the MMAs; a ragged last slab
// takes the guarded loop, out of line.
__device__ __noinline__ float4 sk_slab_mma_ragged(const bf16_t* tile, const bf16_t* xs0, int nstep, bool has_x,
                                                  int lane) {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int jj = 0; jj < nstep; ++jj) {
        const uint4 a0 = lds128(tile + jj * 512 + lane * 8);
        const uint4 a1 = lds128(tile + jj * 512 + 256 + lane * 8);
        const uint4 Bv = has_x ? lds128(xs0 + jj * 32) : make_uint4(0, 0, 0, 0);
        float (&acc)[4] = (jj & 1) ? c1 : c0;
        mma_bf16_16816(acc, a0.x, a1.x, a0.y, a1.y, Bv.x, Bv.y);
        mma_bf16_16816(acc, a0.z, a1.z, a0.w, a1.w, Bv.z, Bv.w);
    }
    return make_float4(c0[0] + c1[0], c0[1] + c1[1], c0[2] + c1[2], c0[3] + c1[3]);
}
__device__ __forceinline__ float4 sk_slab_mma(const bf16_t* tile, const bf16_t* xb, int sg, int nstep, bool has_x,
                                              int lane) {
    const bf16_t* xs0 = xb + sg * GV_SLAB_STEPS * 32;
    if (nstep != GV_SLAB_STEPS) return sk_slab_mma_ragged(tile, xs0, nstep, has_x, lane);
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jj = 0; jj < GV_SLAB_STEPS; ++jj) {
        const uint4 a0 = lds128(tile + jj * 512 + lane * 8);
        const uint4 a1 = lds128(tile + jj * 512 + 256 + lane * 8);
        const uint4 bv = has_x ? lds128(xs0 + jj * 32) : make_uint4(0, 0, 0, 0);
        float (&acc)[4] = (jj & 1) ? c1 : c0;
        mma_bf16_16816(acc, a0.x, a1.x, a0.y, a1.y, bv.x, bv.y);
        mma_bf16_16816(acc, a0.z, a1.z, a0.w, a1.w, bv.z, bv.w);
    }
    return make_float4(c0[0] + c1[0], c0[1] + c1[1], c0[2] + c1[2], c0[3] + c1[3]);
}

// This warp's slabs j in [jb, je) of a phase round (j congruent to `first`
// mod 8): wait, partial sums, release the slot, partials to the partial
// buffer (slab j at pbuf[(j - jb) * 128]).
__device__ __forceinline__ void sk_round_slabs(const SkRing r, const bf16_t* xb, bool has_x, float* pbuf, int gs,
                                            int jb, int je, int first, int nsl, int steps_total,
                                            volatile int* cta_abort, int phase, int lane, unsigned* bar,
                                            int32_t* status, unsigned long long* tslab) {
    const int r8 = lane >> 2, c = lane & 3;
    for (int j = jb + (((first - jb) % SK_CW) + SK_CW) % SK_CW; j < je; j += SK_CW) {
        const int g = gs + j;
        const int slot = g % r.ns;
        if (*cta_abort || !sk_slab_wait(bar, status, tslab, r, g, cta_abort, phase, lane)) break;
        const int sg = j % nsl;
        const int nstep = min(GV_SLAB_STEPS, steps_total - sg * GV_SLAB_STEPS);
        const float4 part = sk_slab_mma(reinterpret_cast<const bf16_t*>(r.ring + slot * SK_SLAB_BYTES), xb, sg,
                                        nstep, has_x, lane);
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&r.empty[slot]);
            if (tslab && blockIdx.x == 0 && g < SK_TRACE_SLABS) tslab[g * 4 + 2] = globaltimer();
        }
        float* pp = pbuf + (j - jb) * SK_PB_SLAB;
        *reinterpret_cast<float2*>(pp + r8 * 8 + 2 * c) = make_float2(part.x, part.y);
        *reinterpret_cast<float2*>(pp + (r8 + 8) * 8 + 2 * c) = make_float2(part.z, part.w);
    }
}

// The GEMV of one phase for this CTA's consumer warps.  gs: the CTA's slab
// sequence number at the phase start (advanced past the phase's slabs); vc:
// the CTA's place in the phase's item order.  Slab j of the phase (slab j % nks
// of item j / nks) goes to warp (gs + j) % 8; the items' slab partials gather
// in the partial buffer a round of items at a time, and item i's warp adds them
// in slab order and runs the epilogue (gv_finish).
template <int EPI>
__device__ void sk_gemv_consume(const SkParams& s, const GemvParams& p, const SkRing& r, const bf16_t* xs,
                                float* pbuf, float* cbuf, GvBest<1>& best, int& gs, int vc,
                                volatile int* cta_abort, int warp, int lane, int phase,
                                unsigned long long* td = nullptr, const float* rpre = nullptr) {
    const int G = gridDim.x;
    const int XS = p.K + GV_PAD;
    const int r8 = lane >> 2, c = lane & 3;
    const bool has_x = r8 < s.M;
    const bf16_t* xb = xs + (has_x ? r8 : 0) * XS + 8 * c;
    const int steps_total = p.K >> 5;
    const int nmine = sk_cta_items(p.n_items, vc);
    const int first = ((warp - gs) % SK_CW + SK_CW) % SK_CW;  // this warp's first phase slab
    const int nsl = p.nks;
    const int R = max(1, s.pb / nsl);  // items per round
    for (int i0 = 0; i0 < nmine; i0 += R) {
        const int i1 = min(nmine, i0 + R);
        sk_round_slabs(r, xb, has_x, pbuf, gs, i0 * nsl, i1 * nsl, first, nsl, steps_total, cta_abort, phase, lane,
                       s.bar, s.status, s.tslab);
        if (td && i0 == 0) td[4] = globaltimer();
        named_bar(1, SK_CT);
        if (td && i0 == 0) td[5] = globaltimer();
        if (!*cta_abort) {
            for (int i = i0 + warp; i < i1; i += SK_CW) {
                float yacc[1][4];
                for (int sl = 0; sl < nsl; ++sl) {
                    const float* pp = pbuf + ((i - i0) * nsl + sl) * SK_PB_SLAB;
                    const float2 lo = *reinterpret_cast<const float2*>(pp + r8 * 8 + 2 * c);
                    const float2 hi = *reinterpret_cast<const float2*>(pp + (r8 + 8) * 8 + 2 * c);
                    if (sl == 0) { yacc[0][0] = lo.x; yacc[0][1] = lo.y; yacc[0][2] = hi.x; yacc[0][3] = hi.y; }
                    else { yacc[0][0] += lo.x; yacc[0][1] += lo.y; yacc[0][2] += hi.x; yacc[0][3] += hi.y; }
                }
                if (EPI == EPI_RESID && rpre && i == warp) {
                    // the residual add of gv_finish, on the rows loaded before the phase
                    const int rb = vc + i * G;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int n = 2 * c + (q & 1), col = rb * GV_ROWS + r8 + ((q & 2) ? 8 : 0);
                        if (n < p.M && col < p.N)
                            reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(rpre[q] + yacc[0][q]);
                    }
                } else {
                    gv_finish<1, EPI>(p, vc + i * G, 0, yacc, lane, cbuf + warp * GV_ROWS * 8, best);
                }
            }
        }
        if (td && i0 == 0) td[6] = globaltimer();
        named_bar(1, SK_CT);  // the partial buffer is reused by the next round
        if (td && i0 == 0) td[7] = globaltimer();
    }
    gs += nmine * nsl;
}

// ------------------------------------------------------------ GDN and attention

// S rows row0..row0+3 of (stream b, head h) of GDN layer ig into registers,
// with the head's A = exp(A_log) and dt_bias.
template <int KPL>
__device__ __forceinline__ float* sk_gdn_rows(const SkParams& s, int l, int ig, int it, float (&S)[GDN_RPW][KPL],
                                              float& A, float& dtb, int lane) {
    constexpr int DK = 32 * KPL;
    const int rg = s.dv / GDN_RPW;
    const int b = it / (s.H * rg), h = (it / rg) % s.H, row0 = (it % rg) * GDN_RPW;
    const bf16_t* const* w = s.layer[l].w;
    A = expf(bf2f(w[HGD_W_A_LOG][h]));
    dtb = bf2f(w[HGD_W_DT_BIAS][h]);
    float* Sbase = s.S + (size_t)ig * s.B * s.H * s.dv * DK + ((int64_t)(b * s.H + h) * s.dv + row0) * DK + lane * KPL;
#pragma unroll
    for (int r = 0; r < GDN_RPW; ++r) ld_vec<KPL>(S[r], Sbase + (int64_t)r * DK);
    return Sbase;
}

// Gated delta rule of GDN item `it` (4 state rows of one stream and head) over
// the call's T rows, on state rows already in S: the arithmetic of k_gdn_layer.
template <int KPL>
__device__ void sk_gdn_item(const SkParams& s, int ig, int it, float (&S)[GDN_RPW][KPL], float* Sbase, float A,
                            float dtb, int lane) {
    constexpr int DK = 32 * KPL;
    const int H = s.H, dv = s.dv, rg = dv / GDN_RPW;
    const int b = it / (H * rg), h = (it / rg) % H, row0 = (it % rg) * GDN_RPW;
    for (int t = 0; t < s.T; ++t) {
        const int64_t row = (int64_t)b * s.T + t;
        const float* pr = s.proj + row * s.proj_ld;
        float qv[KPL], kv[KPL];
        const int hk = h / (H / s.Hk);
        ld_vec<KPL>(qv, pr + (int64_t)hk * DK + lane * KPL);
        ld_vec<KPL>(kv, pr + (int64_t)s.Hk * DK + (int64_t)hk * DK + lane * KPL);
        const float a = pr[s.C + (int64_t)H * dv + h];
        const float braw = pr[s.C + (int64_t)H * dv + H + h];
        float vrow[GDN_RPW], o[GDN_RPW];
        const float* vp = pr + 2 * (int64_t)s.Hk * DK + (int64_t)h * dv + row0;
#pragma unroll
        for (int r = 0; r < GDN_RPW; ++r) vrow[r] = vp[r];
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int e = 0; e < KPL; ++e) { sq = fmaf(qv[e], qv[e], sq); sk = fmaf(kv[e], kv[e], sk); }
        const float qsc = rsqrtf(warp_sum(sq) + 1e-6f), ksc = rsqrtf(warp_sum(sk) + 1e-6f);
#pragma unroll
        for (int e = 0; e < KPL; ++e) { qv[e] = qv[e] * qsc; kv[e] = kv[e] * ksc; }
        const float g = -A * softplus_f(a + dtb);
        const float alpha = expf(g);
        const float beta = sigmoid_f(braw);
        float dl[GDN_RPW];
        gdn_rows_step<KPL>(S, kv, qv, alpha, beta, vrow, o, dl);
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
// Shared memory: ring [ns][8 KB] | xs [M][kmax + 8] bf16 | gains [D] bf16 |
// partial buffer [pb][16][8] f32 | conv scratch [8][16][8] f32 | argmax [8][8] x2 |
// attention scratch [8][32] f32 | full[ns], empty[ns] mbarriers | flags.
struct SkSmem {
    uint8_t* ring; bf16_t* xs; bf16_t* gb[2]; float* pbuf; float* cbuf; float* amax_v; int* amax_i; float* ex;
    uint64_t* full; uint64_t* empty; volatile int* flags;
};

__host__ __device__ inline size_t sk_al128(size_t v) { return (v + 127) & ~(size_t)127; }
__host__ __device__ inline size_t sk_xs_bytes(int M, int kmax) { return sk_al128((size_t)M * (kmax + GV_PAD) * 2); }
__host__ __device__ inline size_t sk_fixed_bytes(int M, int kmax, int D, int pb, int ns) {
    return sk_xs_bytes(M, kmax) + 2 * sk_al128((size_t)D * 2) + (size_t)pb * SK_PB_SLAB * 4 +
           (size_t)SK_CW * GV_ROWS * 8 * 4 + (size_t)SK_CW * 8 * 8 + (size_t)SK_CW * 32 * 4 + (size_t)ns * 16 + 64;
}

__device__ __forceinline__ SkSmem sk_smem(const SkParams& s, uint8_t* base) {
    SkSmem m;
    size_t o = 0;
    m.ring = base; o += (size_t)s.ns * SK_SLAB_BYTES;
    m.xs = reinterpret_cast<bf16_t*>(base + o); o += sk_xs_bytes(s.M, s.kmax);
    m.gb[0] = reinterpret_cast<bf16_t*>(base + o); o += sk_al128((size_t)s.D * 2);
    m.gb[1] = reinterpret_cast<bf16_t*>(base + o); o += sk_al128((size_t)s.D * 2);
    m.pbuf = reinterpret_cast<float*>(base + o); o += (size_t)s.pb * SK_PB_SLAB * 4;
    m.cbuf = reinterpret_cast<float*>(base + o); o += (size_t)SK_CW * GV_ROWS * 8 * 4;
    m.amax_v = reinterpret_cast<float*>(base + o); o += SK_CW * 8 * 4;
    m.amax_i = reinterpret_cast<int*>(base + o); o += SK_CW * 8 * 4;
    m.ex = reinterpret_cast<float*>(base + o); o += SK_CW * 32 * 4;
    m.full = reinterpret_cast<uint64_t*>(base + o); o += (size_t)s.ns * 8;
    m.empty = reinterpret_cast<uint64_t*>(base + o); o += (size_t)s.ns * 8;
    m.flags = reinterpret_cast<volatile int*>(base + o);
    return m;
}

// Gains of phase pid (layer l, phase j of the layer) into gains buffer pid & 1,
// by cp.async, as one committed group (empty if the phase reads none): each
// phase's gains are issued one phase ahead, so they land while the phase
// before runs.
__device__ __forceinline__ void sk_issue_gains(const SkParams& s, const SkSmem& sm, int pid, int l, int j, int tid) {
    if (l <= s.L && j < ((l == s.L) ? 2 : SK_PHASES_PER_LAYER)) {
        int n = 0;
        const bf16_t* g = sk_gains(s, sk_kind(s, l, j), l, n);
        if (g)
            for (int c = tid; c < n / 8; c += SK_CT) cp_async16(((pid & 1) ? sm.gb[1] : sm.gb[0]) + c * 8, g + c * 8);
    }
    cp_async_commit();
}

// KPL: GDN key elements per lane (dk / 32); DPL: attention dims per lane (hd / 32).
template <int KPL, int DPL>
__global__ void __launch_bounds__(SK_THREADS, 1) k_stack(const __grid_constant__ SkParams s) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const SkSmem sm = sk_smem(s, smem);
    volatile int* cta_abort = sm.flags;
    volatile int* seen = sm.flags + 1;  // the last phase whose completion a poller saw
    const SkRing ring{sm.ring, sm.full, sm.empty, s.ns};
    const int G = gridDim.x;

    if (tid == 0) {
        for (int i = 0; i < s.ns; ++i) { mbar_init(&sm.full[i], 1); mbar_init(&sm.empty[i], 1); }
        *cta_abort = 0;
        seen[0] = -1;
        mbar_fence_init();
    }
    __syncthreads();

    // ---------------------------------------------------------------- producer
    // The CTA's slabs of a phase, j = 0 .. nmine * nks - 1 (slab j % nks of item
    // j / nks), go out eight at a time: lane l of the producer warp takes slab
    // j0 + l, waits for its ring slot to be released and issues its bulk copy.
    if (warp == SK_CW) {
        constexpr int PB = 8;  // copies issued together (<= ring slots)
        const uint64_t pol = policy_evict_first();
        int g = 0;  // the CTA's slab sequence number at the start of the batch
        bool ok = true;
        int pid = -1;
        for (int l = 0; l <= s.L && ok; ++l) {
            const int nph = (l == s.L) ? 1 : SK_PHASES_PER_LAYER;
            for (int jph = 0; jph < nph && ok; ++jph) {
                ++pid;
                const int kind = sk_kind(s, l, jph);
                if (!sk_is_gemv(kind)) continue;
                GemvParams p;
                sk_gemv_params(s, kind, l, 0, 0, p);
                const int steps_total = p.K >> 5;
                const int vc = sk_vcta(pid);
                const int J = sk_cta_items(p.n_items, vc) * p.nks;
                for (int j0 = 0; j0 < J && ok; j0 += PB) {
                    const int j = j0 + lane;
                    bool lane_ok = true, sent = false;
                    if (lane < PB && j < J) {
                        const int gj = g + lane;
                        const int slot = gj % s.ns;
                        if (gj >= s.ns && !mbar_wait_sleepy(&sm.empty[slot], (uint32_t)(((gj / s.ns) - 1) & 1),
                                                            cta_abort, 64u)) {
                            // (an abort raised elsewhere reaches this CTA through its consumers' waits)
                            if (!*cta_abort) sk_timeout(s, 3u, (unsigned)pid, (unsigned)gj);
                            lane_ok = false;
                        } else {
                            const int i = j / p.nks, sg = j % p.nks;
                            const int rb = vc + i * G;
                            const int nstep = min(GV_SLAB_STEPS, steps_total - sg * GV_SLAB_STEPS);
                            const uint32_t bytes = (uint32_t)nstep * 1024u;
                            if (s.tslab && blockIdx.x == 0 && gj < SK_TRACE_SLABS) s.tslab[gj * 4] = globaltimer();
                            mbar_arrive_expect_tx(&sm.full[slot], bytes);
                            bulk_g2s(ring.ring + (size_t)slot * SK_SLAB_BYTES,
                                     p.W + gv_tile_elem(rb, sg * GV_SLAB_STEPS, steps_total, 0, 0), bytes,
                                     &sm.full[slot], pol);
                            sent = true;
                        }
                    }
                    ok = __all_sync(0xffffffffu, lane_ok);
                    if (!ok) {
                        // a wait ran out: the copies this batch did send land before the
                        // warp leaves; g stays at the batch start for the drain below
                        if (sent) {
                            const int gj = g + lane;
                            (void)mbar_wait_bounded(&sm.full[gj % s.ns], (uint32_t)((gj / s.ns) & 1), nullptr);
                        }
                        break;
                    }
                    g += min(PB, J - j0);
                }
            }
        }
        // Do not leave while a copy into this CTA's shared memory is in flight:
        // wait for the fills of the last ns slabs issued (a slot whose copy was
        // never issued after a failed wait completed its earlier fill already).
        if (lane == 0)
            for (int q = max(0, g - s.ns); q < g; ++q)
                (void)mbar_wait_bounded(&sm.full[q % s.ns], (uint32_t)((q / s.ns) & 1), nullptr);
        return;
    }

    // --------------------------------------------------------------- consumers
    int gs = 0;       // the CTA's slab sequence number (same in every consumer warp)
    int ig = 0, ia = 0, pid = -1;
    GvBest<1> best;
    best.init();
    sk_issue_gains(s, sm, 0, 0, 0, tid);
    for (int l = 0; l <= s.L; ++l) {
        const int nph = (l == s.L) ? 2 : SK_PHASES_PER_LAYER;
        for (int j = 0; j < nph; ++j) {
            const int kind = sk_kind(s, l, j);
            ++pid;
            if (kind == SK_FINAL) {
                if (blockIdx.x == 0) {
                    const bool live = sk_wait(s, cta_abort, seen, pid - 1);
                    if (live && warp == 0) sk_final(s, lane);
                }
                continue;
            }
            GemvParams p;
            const bool gemv = sk_is_gemv(kind);
            const int vc = sk_vcta(pid);
            int nmine = 0;
            if (gemv) {
                sk_gemv_params(s, kind, l, ig, ia, p);
                nmine = sk_cta_items(p.n_items, vc);
            }
            // work that does not depend on the previous phase: gains, GDN state rows
            float S[GDN_RPW][KPL];
            float* Sbase = nullptr;
            float gA = 0.f, gdtb = 0.f, rpre[4] = {0.f, 0.f, 0.f, 0.f};
            const int gw = warp * G + blockIdx.x, nw = G * SK_CW;
            const int n_gdn = s.B * s.H * (s.dv / GDN_RPW);
            // the next phase's gains go to shared memory asynchronously (this
            // phase's were issued one phase ago; the prologue waits for them)
            if (j + 1 < nph) sk_issue_gains(s, sm, pid + 1, l, j + 1, tid);
            else sk_issue_gains(s, sm, pid + 1, l + 1, 0, tid);
            if (kind == SK_GDN && gw < n_gdn) {
                Sbase = sk_gdn_rows<KPL>(s, l, ig, gw, S, gA, gdtb, lane);
            }
            if (nmine > 0 && (kind == SK_OUT_GDN || kind == SK_OUT_ATT || kind == SK_DOWN)) {
                // the residual rows this warp's first item adds to (written two or
                // more phases ago, stable until this phase writes them)
                const int R = max(1, s.pb / p.nks);
                if (warp < min(R, nmine)) {
                    const int rb = vc + warp * G, r8 = lane >> 2, c = lane & 3;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int n = 2 * c + (q & 1), col = rb * GV_ROWS + r8 + ((q & 2) ? 8 : 0);
                        rpre[q] = (n < s.M && col < p.N) ? bf2f(s.resid[(int64_t)n * s.D + col]) : 0.f;
                    }
                }
            }
            if (kind == SK_IN_ATT) {
                // warm L2 with the key and value chunks of this warp's coming attention partials
                const int n = s.M * s.nq * s.max_chunks;
                const size_t kv_half = (size_t)s.B * s.nkv * s.Lmax * s.hd;
                for (int it = gw; lane == 0 && it < n; it += nw) {
                    const int row = it / (s.nq * s.max_chunks), h = (it / s.max_chunks) % s.nq;
                    const int ch = it % s.max_chunks, b = row / s.T, t = row % s.T;
                    const int P = s.pos[b] + t, key0 = ch * ATTN_CHUNK;
                    if (P < 0 || P >= s.Lmax || key0 > P) continue;
                    const int nk = min(ATTN_CHUNK, P + 1 - key0);
                    const bf16_t* K = s.kv + (size_t)ia * 2 * kv_half +
                                      (((int64_t)b * s.nkv + h / (s.nq / s.nkv)) * s.Lmax + key0) * s.hd;
                    prefetch_l2_bulk(K, (uint32_t)nk * s.hd * 2);
                    prefetch_l2_bulk(K + kv_half, (uint32_t)nk * s.hd * 2);
                }
            }
            const bool live = (pid == 0) ? sk_bar_and(!*cta_abort) : sk_wait(s, cta_abort, seen, pid - 1);
            if (s.trace && blockIdx.x == 0 && tid == 0 && pid < SK_TRACE_SLOTS - 1) s.trace[pid] = globaltimer();
            // per-CTA phase times: wait done, prologue done, GEMV or items done, arrival
            unsigned long long* td = (s.tdetail && tid == 0 && blockIdx.x < SK_TRACE_CTAS)
                                         ? s.tdetail + ((size_t)pid * SK_TRACE_CTAS + blockIdx.x) * 8
                                         : nullptr;
            if (td) td[0] = globaltimer();
            if (live && (!gemv || nmine > 0)) {
                switch (kind) {
                    case SK_IN_GDN: case SK_IN_ATT: case SK_SWIGLU: case SK_HEAD: {
                        const bf16_t* gb = (pid & 1) ? sm.gb[1] : sm.gb[0];
                        if ((kind == SK_SWIGLU || l > 0) && s.D % 256 == 0 && s.D <= 256 * SK_NORM_MAXJ) {
                            sk_pro_resid_rmsnorm(s, sm.xs, gb, warp, lane);
                            break;
                        }
                        if (kind != SK_SWIGLU && l == 0) sk_pro_embed(s, sm.xs);
                        else sk_pro_resid(s, sm.xs);
                        cp_async_wait_prior();
                        named_bar(1, SK_CT);
                        sk_pro_rmsnorm(s, sm.xs, gb, warp, lane);
                        break;
                    }
                    case SK_OUT_GDN:
                        cp_async_wait_prior();
                        named_bar(1, SK_CT);
                        sk_pro_gated(s, p, (pid & 1) ? sm.gb[1] : sm.gb[0], sm.xs, warp, lane);
                        break;
                    case SK_OUT_ATT: sk_pro_copy(s, s.attn, s.nq * s.hd, sm.xs); break;
                    case SK_DOWN: sk_pro_copy(s, s.mlp, s.I, sm.xs); break;
                    default: break;
                }
                named_bar(1, SK_CT);
                if (td) td[1] = globaltimer();
                switch (kind) {
                    case SK_IN_GDN:
                        sk_gemv_consume<EPI_QKV_CONV>(s, p, ring, sm.xs, sm.pbuf, sm.cbuf, best, gs, vc, cta_abort,
                                                      warp, lane, pid, td);
                        break;
                    case SK_IN_ATT:
                        sk_gemv_consume<EPI_ROPE>(s, p, ring, sm.xs, sm.pbuf, sm.cbuf, best, gs, vc, cta_abort, warp,
                                                  lane, pid, td);
                        break;
                    case SK_SWIGLU:
                        sk_gemv_consume<EPI_SWIGLU>(s, p, ring, sm.xs, sm.pbuf, sm.cbuf, best, gs, vc, cta_abort,
                                                    warp, lane, pid, td);
                        break;
                    case SK_HEAD:
                        sk_gemv_consume<EPI_ARGMAX>(s, p, ring, sm.xs, sm.pbuf, sm.cbuf, best, gs, vc, cta_abort,
                                                    warp, lane, pid, td);
                        gv_argmax_cta<1>(p, best, sm.amax_v, sm.amax_i, warp, lane, tid, SK_CW, blockIdx.x, G, true);
                        break;
                    case SK_OUT_GDN: case SK_OUT_ATT: case SK_DOWN:
                        sk_gemv_consume<EPI_RESID>(s, p, ring, sm.xs, sm.pbuf, sm.cbuf, best, gs, vc, cta_abort,
                                                   warp, lane, pid, td, rpre);
                        break;
                    case SK_GDN:
                        for (int it = gw; it < n_gdn; it += nw) {
                            if (it != gw) Sbase = sk_gdn_rows<KPL>(s, l, ig, it, S, gA, gdtb, lane);
                            sk_gdn_item<KPL>(s, ig, it, S, Sbase, gA, gdtb, lane);
                        }
                        break;
                    case SK_PART: {
                        // partials per (row, head, 32-key chunk), one warp each; the last
                        // chunk of a (row, head) to finish queues its merge, which the whole
                        // CTA then runs with one dim per thread
                        volatile int* mlist = reinterpret_cast<volatile int*>(sm.ex);  // count, (row*nq+h, nch)...
                        const int mcap = (SK_CW * 32 - 1) / 2;
                        if (tid == 0) mlist[0] = 0;
                        named_bar(1, SK_CT);
                        const int n = s.M * s.nq * s.max_chunks;
                        const size_t kv_half = (size_t)s.B * s.nkv * s.Lmax * s.hd;
                        const int group = s.nq / s.nkv;
                        for (int it = gw; it < n; it += nw) {
                            const int row = it / (s.nq * s.max_chunks), h = (it / s.max_chunks) % s.nq;
                            const int ch = it % s.max_chunks;
                            const int b = row / s.T, t = row % s.T;
                            const int P = s.pos[b] + t;
                            if (P < 0 || P >= s.Lmax) {  // the merged output of the row is zero
                                if (ch == 0)
                                    for (int d = lane; d < s.hd; d += 32)
                                        s.attn[(int64_t)row * s.nq * s.hd + (int64_t)h * s.hd + d] = 0;
                                continue;
                            }
                            const int key0 = ch * ATTN_CHUNK;
                            if (key0 > P) continue;
                            const int g = h / group;
                            const bf16_t* K = s.kv + (size_t)ia * 2 * kv_half + ((int64_t)b * s.nkv + g) * s.Lmax * s.hd;
                            const float* q = s.qrot + (int64_t)row * s.nq * s.hd + (int64_t)h * s.hd;
                            float* dst = s.part + (((int64_t)row * s.nq + h) * s.max_chunks + ch) * (s.hd + 2);
                            attn_partial_warp_t<DPL>(q, K, K + kv_half, key0, min(ATTN_CHUNK, P + 1 - key0), dst,
                                                     lane);
                            const int nch = P / ATTN_CHUNK + 1;
                            int k = -1;  // this warp's place in the merge queue, or -1
                            if (lane == 0) {
                                __threadfence();
                                const unsigned old = atomicAdd(s.mcnt + row * s.nq + h, 1u);
                                if (old == (unsigned)nch - 1u) {
                                    __threadfence();  // the other chunks' partials are visible from here on
                                    k = atomicAdd(const_cast<int*>(mlist), 1);
                                    if (k < mcap) {
                                        mlist[1 + 2 * k] = row * s.nq + h;
                                        mlist[2 + 2 * k] = nch;
                                    }
                                }
                            }
                            k = __shfl_sync(0xffffffffu, k, 0);
                            if (k >= mcap) {  // queue full: this warp merges the head itself
                                const float* base = s.part + ((int64_t)row * s.nq + h) * s.max_chunks * (s.hd + 2);
                                const float* gate = s.proj + (int64_t)row * s.proj_ld + s.nq * s.hd + (int64_t)h * s.hd;
                                sk_merge_head_t<DPL>(base, nch, gate,
                                                     s.attn + (int64_t)row * s.nq * s.hd + (int64_t)h * s.hd, lane);
                                if (lane == 0) s.mcnt[row * s.nq + h] = 0u;
                            }
                        }
                        named_bar(1, SK_CT);
                        const int nm = min((int)mlist[0], mcap);
                        for (int e = 0; e < nm; ++e) {
                            const int rh = mlist[1 + 2 * e], nch = mlist[2 + 2 * e];
                            const int row = rh / s.nq, h = rh % s.nq, hd = s.hd;
                            const float* base = s.part + (int64_t)rh * s.max_chunks * (hd + 2);
                            const float* gate = s.proj + (int64_t)row * s.proj_ld + s.nq * hd + (int64_t)h * hd;
                            bf16_t* out = s.attn + (int64_t)row * s.nq * hd + (int64_t)h * hd;
                            for (int d = tid; d < hd; d += SK_CT) {
                                // the arithmetic of attn_merge_dim for dim d
                                float Mx = -INFINITY;
#pragma unroll 8
                                for (int c = 0; c < nch; ++c) Mx = fmaxf(Mx, __ldcg(base + (int64_t)c * (hd + 2)));
                                float L = 0.f, acc = 0.f;
#pragma unroll 8
                                for (int c = 0; c < nch; ++c) {
                                    const float* pc = base + (int64_t)c * (hd + 2);
                                    const float w = expf(__ldcg(pc) - Mx);
                                    L = fmaf(w, __ldcg(pc + 1), L);
                                    acc = fmaf(w, __ldcg(pc + 2 + d), acc);
                                }
                                out[d] = f2bf(acc / L * sigmoid_f(gate[d]));
                            }
                            if (tid == 0) s.mcnt[rh] = 0u;  // ready for the next attention layer
                        }
                        break;
                    }
                    default: break;
                }
            } else if (gemv) {
                // keep the slab count in step with the producer (nothing is consumed)
                gs += nmine * p.nks;
            }
            if (td) td[2] = globaltimer();
            // this phase's gains have landed even where the phase read none, so the
            // buffer takes the copy issued two phases on (the next phase's may fly)
            cp_async_wait_prior();
            sk_arrive(s, pid);
            if (td) td[3] = globaltimer();
        }
        if (l < s.L) (sk_attn(s, l) ? ia : ig)++;
    }
    if (s.trace && blockIdx.x == 0 && tid == 0) s.trace[SK_TRACE_SLOTS - 1] = globaltimer();
}

}  // namespace hgd
