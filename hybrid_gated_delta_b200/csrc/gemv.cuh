// gemv.cuh -- weight-streaming BF16 GEMV / small-M GEMM engine for sm_100a.
//
// y[m][n] = sum_k x[m][k] W[n][k]  ("decode_linear_benchmark.md" commit message:
// BF16 GEMV and fused up/gate SwiGLU for decode shapes).  Design for B200:
//  * work is cut into 16-row blocks of the weight matrix and 256-column slabs;
//    a warp owns whole work items (a row block, or one slab of it when the row
//    blocks alone cannot occupy every warp of the GPU);
//  * the warp loads its mma.sync A fragments straight from HBM with 128-bit
//    non-allocating loads (L2 evict-first: weights are read once per step),
//    eight 32-column steps in flight per warp in a rolling register pipeline:
//    no shared-memory staging, no copy engine on the critical path.  Columns are
//    taken in a per-thread permuted order (the same permutation for the weight
//    and the token fragments, so each MMA still forms the exact dot product),
//    which makes every fragment a contiguous 16-byte load;
//  * mma.sync m16n8k16 with the weight rows as the MMA M dimension and up to 32
//    token rows as N (swap-AB), fp32 accumulation in two chains (even / odd
//    steps); the token rows sit in shared memory, padded so fragment loads are
//    conflict free;
//  * every output is the sum, in slab order, of per-slab partials (chain 0 +
//    chain 1): its arithmetic depends on K alone, not on M, N, the grid, the SM
//    count or how slabs are spread over warps.  Split slabs meet in a workspace
//    and the last arriver adds them in slab order (no floating-point atomics);
//  * fused prologues (RMSNorm of the residual stream, embedding gather, gated
//    RMSNorm) and epilogues (fp32 / bf16 store, residual add, SwiGLU, argmax,
//    the causal conv of the GDN q|k|v channels);
//  * programmatic dependent launch: each warp issues its first weight loads
//    before griddepcontrol.wait, overlapping the previous kernel's tail.
#pragma once

#include "common.cuh"

namespace hgd {

constexpr int GV_CW = 8;                       // warps per CTA
constexpr int GV_WARPS = GV_CW;
constexpr int GV_THREADS = GV_CW * 32;
constexpr int GV_ROWS = 16;
constexpr int GV_KS = 256;                     // slab width
constexpr int GV_SLAB_STEPS = GV_KS / 32;      // 32-column steps per slab
constexpr int GV_PAD = 8;                      // bf16 elements of padding per token row
constexpr int GV_SMEM_LIMIT = 227 * 1024;

enum GvPrologue { PRO_COPY = 0, PRO_RMSNORM = 1, PRO_EMBED_RMSNORM = 2, PRO_GATED_NORM = 3 };
enum GvEpilogue { EPI_F32 = 0, EPI_BF16 = 1, EPI_RESID = 2, EPI_SWIGLU = 3, EPI_ARGMAX = 4, EPI_QKV_CONV = 5,
                  EPI_ROPE = 6 };
constexpr int GV_CONV_K = 4;  // conv width of the fused conv epilogue

struct GemvParams {
    const bf16_t* W;   // [N][K]; SwiGLU: gate weights [I][K]; packed: the tiles (see gv_tile)
    const bf16_t* W2;  // SwiGLU: up weights [I][K] (unpacked only)
    int packed;        // 1: W holds the fragment-ordered tiles of the (virtual) matrix
    int N, K, M;       // N output features, M token rows of this launch
    int nks;           // slabs per row block (K / 256 rounded up)
    int n_rowblk;      // row blocks (16 rows; SwiGLU: 8 gate + 8 up rows)
    int split;         // 1: one slab per work item, partials through the workspace
    int n_items;       // n_rowblk * (split ? nks : 1)
    int x_bytes;       // bytes of the token rows in shared memory
    // prologue
    const bf16_t* x; int64_t x_ld;         // COPY: [M][x_ld]; RMSNORM: residual rows
    const bf16_t* norm_w; float eps;       // RMSNORM gains [K]
    const int32_t* tokens;                 // EMBED: token per row
    const bf16_t* embed; int vocab;        // EMBED: [vocab][K]
    bf16_t* resid_out; int64_t resid_out_ld;  // EMBED: residual rows written by CTA 0
    const float* o; int64_t o_ld;          // GATED: o rows [M][o_ld]
    const float* z; int64_t z_ld;          // GATED: z rows (fp32, rounded to bf16 here)
    const bf16_t* gnorm_w; int gn_d;       // GATED: gain [gn_d], head width gn_d
    // epilogue
    void* y; int64_t y_ld;                 // F32 / BF16 / RESID / SWIGLU output rows
    const bf16_t* resid; int64_t resid_ld; // RESID: residual rows (may alias y)
    float* logits; int64_t logits_ld;      // ARGMAX: optional logits rows
    float* best_v; int32_t* best_i;        // ARGMAX: [M][gridDim.x] partials
    // split-K workspace: partials [n_rowblk * nks][16][ws_mp] fp32, counters [n_rowblk]
    float* ws_part; int32_t* ws_cnt; int ws_mp;
    // QKV_CONV: outputs < conv_C are channels of the depthwise causal conv (width 4,
    // SiLU): y = silu(sum_j w[c][j] u_j) over the kept tail and the new value, the
    // tail [B][3][conv_C] shifted in place, tail records [B][T][3][conv_C] (or null).
    // Token row m of this launch is stream (m0 + m) / conv_T, row (m0 + m) % conv_T.
    const bf16_t* conv_w; float* conv_tail; float* conv_rec; int conv_C, conv_T, m0;
    float* conv_xlog;  // QKV_CONV: the conv input of each row [B][T][conv_C] (a verify window's log), or null
    // ROPE: the attention in-projection, packed with rope_src_row's row order:
    // q rows are rotated and stored fp32 in rope_q [M][nq*hd]; gate rows go to y
    // (fp32) at column nq*hd + g; k rows are rotated and v rows copied into the
    // bf16 caches [B][nkv][Lmax][hd] at position pos[b] + t (row m0 + m is stream
    // (m0 + m) / conv_T, row (m0 + m) % conv_T).
    int rope_nq, rope_nkv, rope_hd, rope_Lmax; double rope_inv1;  // inv1 = base^(-2/hd)
    float* rope_q; bf16_t* rope_k; bf16_t* rope_v; const int32_t* rope_pos;
    int32_t* status;
};

__host__ __device__ inline int gv_align16(int v) { return (v + 15) & ~15; }
__host__ __device__ inline int gv_slabs(int K) { return (K + GV_KS - 1) / GV_KS; }

// Source row of tile row i (0..15) of row block rb; nullptr if past the end.
__device__ __forceinline__ const bf16_t* gv_row(const GemvParams& p, bool swi, int rb, int i) {
    if (swi) {
        const int r = rb * 8 + (i & 7);
        if (r >= p.N) return nullptr;
        return (i < 8 ? p.W : p.W2) + (int64_t)r * p.K;
    }
    const int r = rb * GV_ROWS + i;
    if (r >= p.N) return nullptr;
    return p.W + (int64_t)r * p.K;
}

// Fragment-ordered weight layout.  The matrix (for SwiGLU the virtual matrix
// whose row block rb holds gate rows 8rb..8rb+7 then up rows 8rb..8rb+7) is cut
// into 16-row x 32-column tiles, row block major; tile (rb, step) is 512 bf16 at
// element (rb * K/32 + step) * 512.  Within a tile, lane l = 4*r8 + c of a warp
// owns elements [8l, 8l+8) (row r8) and [256 + 8l, 256 + 8l + 8) (row r8 + 8),
// each the eight columns step*32 + 8c .. +7 of its row: one warp-wide 16-byte
// load per half-tile reads 512 contiguous bytes.  Rows past the matrix are zero.
__host__ __device__ inline int64_t gv_tile_elem(int64_t rb, int step, int steps, int half, int lane) {
    return ((rb * steps + step) * 512) + half * 256 + lane * 8;
}

// Offset (elements) of the 16-byte chunk cc (columns 8cc..8cc+7) of row n of a
// packed plain matrix with `steps` = K/32 column steps.
__host__ __device__ inline int64_t gv_packed_chunk(int64_t n, int cc, int steps) {
    const int i = (int)(n & 15);
    return gv_tile_elem(n >> 4, cc >> 2, steps, i >> 3, ((i & 7) << 2) | (cc & 3));
}

// Row order of the packed attention in-projection [q | gate | k | v] (rows of
// nq*hd, nq*hd, nkv*hd, nkv*hd): within each q and k head the 16-row block j
// holds dims 8j..8j+7 in its rows 0..7 and their rotate-half partners
// hd/2 + 8j .. +7 in rows 8..15, so one lane's accumulators hold both halves of
// a RoPE pair; gate and v rows keep their order.  Returns the source row of
// virtual row v (a bijection on [0, 2*nq*hd + 2*nkv*hd)).
__host__ __device__ inline int64_t rope_src_row(int64_t v, int nq, int nkv, int hd) {
    const int64_t qw = (int64_t)nq * hd, kw = (int64_t)nkv * hd;
    int64_t base, w;
    if (v < qw) { base = 0; w = v; }
    else if (v < 2 * qw) return v;
    else if (v < 2 * qw + kw) { base = 2 * qw; w = v - 2 * qw; }
    else return v;
    const int64_t head = w / hd;
    const int r = (int)(w % hd), j = r >> 4, i16 = r & 15;
    const int dim = (i16 < 8) ? 8 * j + i16 : hd / 2 + 8 * j + (i16 - 8);
    return base + head * hd + dim;
}

// sin and cos of the RoPE angle of dim pair i at position P: the angle
// P * base^(-2i/hd) in double, with base^(-2i/hd) = inv1^i (inv1 = base^(-2/hd),
// computed once in double on the host; the power by repeated squaring in
// double, relative error ~1e-15), reduced to [-pi, pi] in double, then the fp32
// sine and cosine of the reduced angle.
__device__ __forceinline__ void rope_sincos(int P, int i, double inv1, float* sn, float* cs) {
    double inv = 1.0, b = inv1;
    for (int e = i; e; e >>= 1) {
        if (e & 1) inv *= b;
        b *= b;
    }
    const double th = (double)P * inv;
    const double tw = 6.283185307179586476925286766559, itw = 0.15915494309189533576888376337251;
    const float r = (float)(th - tw * rint(th * itw));
    sincosf(r, sn, cs);
}

__device__ __forceinline__ float ld_cg(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// 16-byte streaming load of weights: not allocated in L1, evict-first in L2.
__device__ __forceinline__ uint4 ldg_stream(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// ----------------------------------------------------------------- prologues
// Fill xs[MP][K+PAD] (bf16) with this launch's token rows; rows >= M are zero.
// Every CTA computes the same values in the same order.
template <int MP, int PRO>
__device__ __forceinline__ void gv_prologue(const GemvParams& p, bf16_t* xs, int ctid, int cwarp,
                                            int lane, float* scratch) {
    const int K = p.K;
    const int XS = K + GV_PAD;
    if (PRO == PRO_COPY) {
        const int cpr = K / 8;  // 16-byte chunks per row
        for (int e = ctid; e < MP * cpr; e += GV_WARPS * 32) {
            const int m = e / cpr, c = e % cpr;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < p.M) v = *reinterpret_cast<const uint4*>(p.x + m * p.x_ld + c * 8);
            *reinterpret_cast<uint4*>(xs + m * XS + c * 8) = v;
        }
        return;
    }
    if (PRO == PRO_RMSNORM || PRO == PRO_EMBED_RMSNORM) {
        // One warp per token row: sum of squares (lane-strided 8-element chunks,
        // then a butterfly), then x * rsqrt(mean + eps) * w rounded to bf16.
        for (int m = cwarp; m < MP; m += GV_WARPS) {
            bf16_t* dst = xs + m * XS;
            if (m >= p.M) {
                for (int c = lane; c < K / 8; c += 32)
                    *reinterpret_cast<uint4*>(dst + c * 8) = make_uint4(0, 0, 0, 0);
                continue;
            }
            const bf16_t* src;
            if (PRO == PRO_EMBED_RMSNORM) {
                const int tok = p.tokens[m];
                if (tok < 0 || tok >= p.vocab) {  // reject, never read out of bounds
                    if (lane == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
                    for (int c = lane; c < K / 8; c += 32) {
                        *reinterpret_cast<uint4*>(dst + c * 8) = make_uint4(0, 0, 0, 0);
                        if (blockIdx.x == 0)
                            *reinterpret_cast<uint4*>(p.resid_out + m * p.resid_out_ld + c * 8) = make_uint4(0, 0, 0, 0);
                    }
                    continue;
                }
                src = p.embed + (int64_t)tok * K;
            } else {
                src = p.x + m * p.x_ld;
            }
            // 16-byte chunk c of the source row (the embedding is stored packed)
            auto chunk = [&](int c) -> const uint4* {
                if (PRO == PRO_EMBED_RMSNORM)
                    return reinterpret_cast<const uint4*>(p.embed + gv_packed_chunk(p.tokens[m], c, K >> 5));
                return reinterpret_cast<const uint4*>(src + c * 8);
            };
            float ss = 0.f;
            for (int c = lane; c < K / 8; c += 32) {
                const uint4 v = *chunk(c);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float a = bf_lo(w4[q]), b = bf_hi(w4[q]);
                    ss = fmaf(a, a, ss);
                    ss = fmaf(b, b, ss);
                }
            }
            ss = warp_sum(ss);
            const float r = rsqrtf(ss / (float)K + p.eps);
            for (int c = lane; c < K / 8; c += 32) {
                const uint4 v = *chunk(c);
                const uint4 g = *reinterpret_cast<const uint4*>(p.norm_w + c * 8);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                const uint32_t g4[4] = {g.x, g.y, g.z, g.w};
                uint32_t o4[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    o4[q] = pack_bf2(bf_lo(w4[q]) * r * bf_lo(g4[q]), bf_hi(w4[q]) * r * bf_hi(g4[q]));
                *reinterpret_cast<uint4*>(dst + c * 8) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                if (PRO == PRO_EMBED_RMSNORM && blockIdx.x == 0)
                    *reinterpret_cast<uint4*>(p.resid_out + m * p.resid_out_ld + c * 8) = v;
            }
        }
        return;
    }
    if (PRO == PRO_GATED_NORM) {
        // Per token row and head of width d: o * rsqrt(mean(o^2)+eps) * w * silu(bf16(z)).
        const int d = p.gn_d;
        const int nh = K / d;
        for (int e = cwarp; e < MP * nh; e += GV_WARPS) {
            const int m = e / nh, h = e % nh;
            bf16_t* dst = xs + m * XS + h * d;
            if (m >= p.M) {
                for (int i = lane; i < d; i += 32) dst[i] = 0;
                continue;
            }
            const float* orow = p.o + m * p.o_ld + h * d;
            const float* zrow = p.z + m * p.z_ld + h * d;
            float ss = 0.f;
            for (int i = lane; i < d; i += 32) ss = fmaf(orow[i], orow[i], ss);
            ss = warp_sum(ss);
            const float r = rsqrtf(ss / (float)d + p.eps);
            for (int i = lane; i < d; i += 32) {
                const float zb = bf2f(f2bf(zrow[i]));
                dst[i] = f2bf(orow[i] * r * bf2f(p.gnorm_w[i]) * silu_f(zb));
            }
        }
        (void)scratch;
        return;
    }
}

// -------------------------------------------------------------------- kernel
// One work item of a warp: row block rb, slabs [s0, s1).
struct GvItem { int rb, s0, s1; };

__device__ __forceinline__ bool gv_item(const GemvParams& p, int slot, int i, GvItem* it) {
    const int u = slot + i * gridDim.x * GV_CW;
    if (u >= p.n_items) return false;
    if (p.split) { it->rb = u / p.nks; it->s0 = u % p.nks; it->s1 = it->s0 + 1; }
    else { it->rb = u; it->s0 = 0; it->s1 = p.nks; }
    return true;
}

// Running argmax of a thread's tokens (nt*8 + 2c + h) over the rows it has seen.
template <int NT>
struct GvBest {
    float v[NT][2];
    int i[NT][2];
    bool nan;
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) { v[nt][0] = v[nt][1] = -INFINITY; i[nt][0] = i[nt][1] = 0x7fffffff; }
        nan = false;
    }
};

// A finished slab partial (split) or row-block sum (unsplit) of row block rb:
// in split mode add it to the workspace and, in the last of the row block's
// slabs to arrive, add all partials in slab order; then run the epilogue.
// `cb` is this warp's [16][MP] shared scratch (conv epilogue).
template <int NT, int EPI>
__device__ __forceinline__ void gv_finish(const GemvParams& p, int rb, int s_item, float (&yacc)[NT][4],
                                          int lane, float* cb, GvBest<NT>& best) {
    constexpr int MP = 8 * NT;
    const int r8 = lane >> 2, c = lane & 3;
        bool finish = true;
        if (p.split) {
            // slab partial -> workspace; the last of the row block's slabs adds them in order
            float* wp = p.ws_part + ((int64_t)(rb * p.nks + s_item) * GV_ROWS) * p.ws_mp;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n0 = nt * 8 + 2 * c;
                wp[r8 * p.ws_mp + n0] = yacc[nt][0];
                wp[r8 * p.ws_mp + n0 + 1] = yacc[nt][1];
                wp[(r8 + 8) * p.ws_mp + n0] = yacc[nt][2];
                wp[(r8 + 8) * p.ws_mp + n0 + 1] = yacc[nt][3];
            }
            __threadfence();
            __syncwarp();
            int old = 0;
            if (lane == 0) old = atomicAdd(&p.ws_cnt[rb], 1);
            old = __shfl_sync(0xffffffffu, old, 0);
            finish = (old == p.nks - 1);
            if (finish) {
                __threadfence();
                // partials in slab order; L2-only loads the compiler may issue ahead
#pragma unroll 4
                for (int j = 0; j < p.nks; ++j) {
                    const float* pp = p.ws_part + ((int64_t)(rb * p.nks + j) * GV_ROWS) * p.ws_mp;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int n0 = nt * 8 + 2 * c;
                        const float2 lo = __ldcg(reinterpret_cast<const float2*>(pp + r8 * p.ws_mp + n0));
                        const float2 hi = __ldcg(reinterpret_cast<const float2*>(pp + (r8 + 8) * p.ws_mp + n0));
                        const float v0 = lo.x, v1 = lo.y, v2 = hi.x, v3 = hi.y;
                        if (j == 0) { yacc[nt][0] = v0; yacc[nt][1] = v1; yacc[nt][2] = v2; yacc[nt][3] = v3; }
                        else { yacc[nt][0] += v0; yacc[nt][1] += v1; yacc[nt][2] += v2; yacc[nt][3] += v3; }
                    }
                }
                if (lane == 0) p.ws_cnt[rb] = 0;  // leave the workspace ready for the next call
            }
        }
        if (!finish) return;
        // ----------------------------------------------------------- epilogue
        if (EPI == EPI_QKV_CONV) {
            // Gather the 16 x MP tile in shared memory; lane l < 16 then runs the conv
            // of channel rb*16 + l over the launch's token rows in order.  The row
            // block (hence the channel and its tail) belongs to this warp alone.
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n0 = nt * 8 + 2 * c;
                cb[r8 * MP + n0] = yacc[nt][0];
                cb[r8 * MP + n0 + 1] = yacc[nt][1];
                cb[(r8 + 8) * MP + n0] = yacc[nt][2];
                cb[(r8 + 8) * MP + n0 + 1] = yacc[nt][3];
            }
            __syncwarp();
            const int ch = rb * GV_ROWS + lane;
            if (lane < GV_ROWS && ch < p.N) {
                float* yrow = reinterpret_cast<float*>(p.y);
                if (ch >= p.conv_C) {
                    for (int m = 0; m < p.M; ++m) yrow[m * p.y_ld + ch] = cb[lane * MP + m];
                } else {
                    float w[GV_CONV_K], tl[GV_CONV_K - 1];
#pragma unroll
                    for (int j = 0; j < GV_CONV_K; ++j) w[j] = bf2f(p.conv_w[(int64_t)ch * GV_CONV_K + j]);
                    int cur_b = -1;
                    for (int m = 0; m < p.M; ++m) {
                        const int gm = p.m0 + m, b = gm / p.conv_T, t = gm % p.conv_T;
                        float* tb = p.conv_tail + (int64_t)b * (GV_CONV_K - 1) * p.conv_C + ch;
                        if (b != cur_b) {
#pragma unroll
                            for (int j = 0; j < GV_CONV_K - 1; ++j) tl[j] = tb[(int64_t)j * p.conv_C];
                            cur_b = b;
                        }
                        const float xv = cb[lane * MP + m];
                        if (p.conv_xlog) p.conv_xlog[((int64_t)b * p.conv_T + t) * p.conv_C + ch] = xv;
                        float acc = 0.f;
#pragma unroll
                        for (int j = 0; j < GV_CONV_K - 1; ++j) acc = fmaf(w[j], tl[j], acc);
                        acc = fmaf(w[GV_CONV_K - 1], xv, acc);
                        yrow[m * p.y_ld + ch] = silu_f(acc);
#pragma unroll
                        for (int j = 0; j + 1 < GV_CONV_K - 1; ++j) tl[j] = tl[j + 1];
                        tl[GV_CONV_K - 2] = xv;
                        if (p.conv_rec) {
                            float* rr = p.conv_rec + ((int64_t)b * p.conv_T + t) * (GV_CONV_K - 1) * p.conv_C + ch;
#pragma unroll
                            for (int j = 0; j < GV_CONV_K - 1; ++j) rr[(int64_t)j * p.conv_C] = tl[j];
                        }
                        if (m == p.M - 1 || t == p.conv_T - 1) {
#pragma unroll
                            for (int j = 0; j < GV_CONV_K - 1; ++j) tb[(int64_t)j * p.conv_C] = tl[j];
                        }
                    }
                }
            }
            __syncwarp();
        } else if (EPI == EPI_ROPE) {
            const int hd = p.rope_hd, half = hd >> 1, hb = hd >> 4;  // 16-row blocks per head
            const int qrb = p.rope_nq * hb, krb = p.rope_nkv * hb, qw = p.rope_nq * hd;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int n = nt * 8 + 2 * c + h2;
                    if (n >= p.M) continue;
                    const float a = yacc[nt][h2], bb = yacc[nt][2 + h2];  // rows r8 and r8 + 8
                    const int gm = p.m0 + n, b = gm / p.conv_T, t = gm % p.conv_T;
                    const int P = p.rope_pos[b] + t;
                    const bool bad = P < 0 || P >= p.rope_Lmax;
                    if (rb >= 2 * qrb + krb) {  // value rows: appended to the V cache
                        if (bad) continue;
                        const int vc = (rb - 2 * qrb - krb) * GV_ROWS + r8;
                        const int g = vc / hd, d = vc % hd;  // vc and vc + 8 share a head (hd % 16 == 0)
                        bf16_t* vo = p.rope_v + (((int64_t)b * p.rope_nkv + g) * p.rope_Lmax + P) * hd;
                        vo[d] = f2bf(a);
                        vo[d + 8] = f2bf(bb);
                    } else if (rb >= qrb && rb < 2 * qrb) {  // output-gate rows
                        const int gc = (rb - qrb) * GV_ROWS + r8;
                        float* y = reinterpret_cast<float*>(p.y) + (int64_t)n * p.y_ld + qw;
                        y[gc] = a;
                        y[gc + 8] = bb;
                    } else {  // q or k rows: the rotate-half pair (i, i + hd/2)
                        const bool isk = rb >= qrb;
                        const int rr = isk ? rb - 2 * qrb : rb;
                        const int head = rr / hb, i = (rr % hb) * 8 + r8;
                        if (bad) {
                            if (isk) set_status(p.status, HGD_ERR_INVALID_ARG);
                            continue;
                        }
                        float sn, cs;
                        rope_sincos(P, i, p.rope_inv1, &sn, &cs);
                        const float x0 = a * cs - bb * sn, x1 = bb * cs + a * sn;
                        if (!isk) {
                            float* qo = p.rope_q + (int64_t)n * qw + (int64_t)head * hd;
                            qo[i] = x0;
                            qo[i + half] = x1;
                        } else {
                            bf16_t* ko = p.rope_k + (((int64_t)b * p.rope_nkv + head) * p.rope_Lmax + P) * hd;
                            ko[i] = f2bf(x0);
                            ko[i + half] = f2bf(x1);
                        }
                    }
                }
            }
        } else {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int n0 = nt * 8 + 2 * c;  // tokens n0, n0 + 1; rows r8, r8 + 8
            if (EPI == EPI_SWIGLU) {
                const int col = rb * 8 + r8;
                if (col < p.N) {
                    bf16_t* h = reinterpret_cast<bf16_t*>(p.y);
                    if (n0 < p.M) h[n0 * p.y_ld + col] = f2bf(silu_f(yacc[nt][0]) * yacc[nt][2]);
                    if (n0 + 1 < p.M) h[(n0 + 1) * p.y_ld + col] = f2bf(silu_f(yacc[nt][1]) * yacc[nt][3]);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int n = n0 + (q & 1);
                    const int col = rb * GV_ROWS + r8 + ((q & 2) ? 8 : 0);
                    if (n >= p.M || col >= p.N) continue;
                    const float v = yacc[nt][q];
                    if (EPI == EPI_F32) {
                        reinterpret_cast<float*>(p.y)[n * p.y_ld + col] = v;
                    } else if (EPI == EPI_BF16) {
                        reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(v);
                    } else if (EPI == EPI_RESID) {
                        const float base = bf2f(p.resid[n * p.resid_ld + col]);
                        reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(base + v);
                    } else {  // EPI_ARGMAX
                        if (p.logits) p.logits[n * p.logits_ld + col] = v;
                        if (v != v) best.nan = true;
                        else if (v > best.v[nt][q & 1] || (v == best.v[nt][q & 1] && col < best.i[nt][q & 1])) {
                            best.v[nt][q & 1] = v;
                            best.i[nt][q & 1] = col;
                        }
                    }
                }
            }
        }
        }
}

// The RMSNorm input of a projection for calls of many token rows, once per row
// instead of in every CTA's prologue: the arithmetic of the PRO_RMSNORM /
// PRO_EMBED_RMSNORM prologue, one warp per row, into out [M][out_ld] (bf16).
// EMBED: the row is the token's (packed) embedding row, also written to the
// residual; a token outside the vocabulary gives zero rows and
// HGD_ERR_INVALID_ARG.
struct NormRowsParams {
    const bf16_t* x; int64_t x_ld;
    const int32_t* tokens; const bf16_t* embed; int vocab;
    bf16_t* resid_out; int64_t resid_out_ld;
    const bf16_t* norm_w; float eps;
    bf16_t* out; int64_t out_ld;
    int M, K;
    int32_t* status;
    int pack_ntp;  // > 0: out holds the rows packed for the tensor-core GEMM (tc_x_elem, NTp rows)
};
template <bool EMBED>
__global__ void __launch_bounds__(256) k_norm_rows(const __grid_constant__ NormRowsParams p) {
    pdl_launch();
    pdl_wait();
    const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (m >= p.M) return;
    const int K = p.K;
    auto dst = [&](int c) -> bf16_t* {
        return p.pack_ntp ? p.out + tc_x_elem(m, c * 8, p.pack_ntp) : p.out + m * p.out_ld + c * 8;
    };
    int tok = 0;
    if (EMBED) {
        tok = p.tokens[m];
        if (tok < 0 || tok >= p.vocab) {
            if (lane == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
            for (int c = lane; c < K / 8; c += 32) {
                *reinterpret_cast<uint4*>(dst(c)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(p.resid_out + m * p.resid_out_ld + c * 8) = make_uint4(0, 0, 0, 0);
            }
            return;
        }
    }
    auto chunk = [&](int c) -> uint4 {
        if (EMBED) return *reinterpret_cast<const uint4*>(p.embed + gv_packed_chunk(tok, c, K >> 5));
        return *reinterpret_cast<const uint4*>(p.x + m * p.x_ld + c * 8);
    };
    // one row chunk c (8 elements) into the sum of squares, in the row's order
    auto sumsq = [](const uint4& v, float ss) {
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = bf_lo(w4[q]), b = bf_hi(w4[q]);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
        return ss;
    };
    auto emit = [&](int c, const uint4& v, const uint4& g, float r) {
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        const uint32_t g4[4] = {g.x, g.y, g.z, g.w};
        uint32_t o4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o4[q] = pack_bf2(bf_lo(w4[q]) * r * bf_lo(g4[q]), bf_hi(w4[q]) * r * bf_hi(g4[q]));
        *reinterpret_cast<uint4*>(dst(c)) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        if (EMBED) *reinterpret_cast<uint4*>(p.resid_out + m * p.resid_out_ld + c * 8) = v;
    };
    // rows of up to NR * 256 elements are read once, into registers; longer rows twice
    constexpr int NR = 8;
    auto gain = [&](int c) { return *reinterpret_cast<const uint4*>(p.norm_w + c * 8); };
    if (K / 8 <= NR * 32) {
        uint4 xr[NR], gr[NR];  // the row and its gains, loaded together
#pragma unroll
        for (int u = 0; u < NR; ++u)
            if (lane + 32 * u < K / 8) { xr[u] = chunk(lane + 32 * u); gr[u] = gain(lane + 32 * u); }
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < NR; ++u)
            if (lane + 32 * u < K / 8) ss = sumsq(xr[u], ss);
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)K + p.eps);
#pragma unroll
        for (int u = 0; u < NR; ++u)
            if (lane + 32 * u < K / 8) emit(lane + 32 * u, xr[u], gr[u], r);
        return;
    }
    float ss = 0.f;
    for (int c = lane; c < K / 8; c += 32) ss = sumsq(chunk(c), ss);
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)K + p.eps);
    for (int c = lane; c < K / 8; c += 32) emit(c, chunk(c), gain(c), r);
}

// The GDN out-projection's input for calls of many token rows, computed once per
// (token row, head) instead of in every CTA's prologue: the arithmetic of the
// PRO_GATED_NORM prologue, one warp per (row, head), into u [M][u_ld] (bf16).
struct GatedNormParams {
    const float* o; int64_t o_ld;
    const float* z; int64_t z_ld;
    const bf16_t* w;
    bf16_t* u; int64_t u_ld;
    int M, nh, d;
    float eps;
    int pack_ntp;  // > 0: u holds the rows packed for the tensor-core GEMM (tc_x_elem, NTp rows)
};
__global__ void __launch_bounds__(256) k_gated_norm(const __grid_constant__ GatedNormParams p) {
    pdl_launch();
    pdl_wait();
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (e >= p.M * p.nh) return;
    const int m = e / p.nh, h = e % p.nh, d = p.d;
    gated_norm_warp(p.o + m * p.o_ld + h * d, p.z + m * p.z_ld + h * d, p.w, d, p.eps, lane, [&](int i, bf16_t v) {
        if (p.pack_ntp) p.u[tc_x_elem(m, h * d + i, p.pack_ntp)] = v;
        else p.u[m * p.u_ld + h * d + i] = v;
    });
}

// Per-CTA argmax partials: reduce each token over the row lanes of every warp,
// then over the warps (`bar` synchronises the nthreads consumer threads).
template <int NT>
__device__ __forceinline__ void gv_argmax_cta(const GemvParams& p, GvBest<NT>& best, float* amax_v, int* amax_i,
                                              int warp, int lane, int tid, int nwarps, int cta, int ncta,
                                              bool named) {
    constexpr int MP = 8 * NT;
    const int r8 = lane >> 2, c = lane & 3;
    const bool any_nan = __any_sync(0xffffffffu, best.nan);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float bv = best.v[nt][h];
            int bi = best.i[nt][h];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if (r8 == 0) {
                amax_v[warp * MP + nt * 8 + 2 * c + h] = bv;
                amax_i[warp * MP + nt * 8 + 2 * c + h] = any_nan ? -1 : bi;
            }
        }
    if (named) named_bar(1, nwarps * 32); else __syncthreads();
    if (tid < p.M) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        bool nan_cta = false;
        for (int w = 0; w < nwarps; ++w) {
            const float v = amax_v[w * MP + tid];
            const int i = amax_i[w * MP + tid];
            if (i < 0) nan_cta = true;
            else if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
        p.best_v[tid * ncta + cta] = bv;
        p.best_i[tid * ncta + cta] = nan_cta ? -1 : bi;
    }
}

template <int NT, int PRO, int EPI>
__global__ void __launch_bounds__(GV_THREADS, (NT >= 4) ? 1 : 2) k_gemv(const __grid_constant__ GemvParams p) {
    constexpr int MP = 8 * NT;
    constexpr int NB = 8;  // 32-column steps in flight per warp
    constexpr bool SWI = (EPI == EPI_SWIGLU);
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = p.K;
    const int XS = K + GV_PAD;
    bf16_t* xs = reinterpret_cast<bf16_t*>(smem);
    float* amax_v = reinterpret_cast<float*>(smem + p.x_bytes);
    int* amax_i = reinterpret_cast<int*>(amax_v + GV_CW * MP);
    float* cbuf = reinterpret_cast<float*>(amax_i + GV_CW * MP);  // [CW][16][MP] (QKV_CONV)

    pdl_launch();
    const uint64_t pol = policy_evict_first();
    const int r8 = lane >> 2, c = lane & 3;
    const int slot = warp * gridDim.x + blockIdx.x;
    const int steps_total = K >> 5;

    // rolling register pipeline of A fragments (rows r8 and r8+8, 16 bytes each)
    uint4 A0[NB], A1[NB];
    const bf16_t* row_lo = nullptr;   // unpacked: the two rows; packed: the row block's tiles
    const bf16_t* row_hi = nullptr;
    auto load_step = [&](int j, int step) {
        if (step < steps_total) {
            if (p.packed) {
                A0[j] = ldg_stream(row_lo + step * 512, pol);
                A1[j] = ldg_stream(row_lo + step * 512 + 256, pol);
            } else {
                const int k = step * 32 + 8 * c;
                A0[j] = row_lo ? ldg_stream(row_lo + k, pol) : make_uint4(0, 0, 0, 0);
                A1[j] = row_hi ? ldg_stream(row_hi + k, pol) : make_uint4(0, 0, 0, 0);
            }
        }
    };
    auto set_rows = [&](int rb) {
        if (p.packed) {
            row_lo = p.W + gv_tile_elem(rb, 0, steps_total, 0, lane);
        } else {
            row_lo = gv_row(p, SWI, rb, r8);
            row_hi = gv_row(p, SWI, rb, r8 + 8);
        }
    };
    GvItem it;
    bool have = gv_item(p, slot, 0, &it);
    if (have) {  // weights never depend on the previous kernel: start streaming now
        set_rows(it.rb);
#pragma unroll
        for (int j = 0; j < NB; ++j) load_step(j, it.s0 * GV_SLAB_STEPS + j);
    }

    pdl_wait();
    gv_prologue<MP, PRO>(p, xs, tid, warp, lane, nullptr);
    __syncthreads();

    GvBest<NT> best;
    best.init();
    const bf16_t* xb = xs + r8 * XS + 8 * c;
    float* cb = cbuf + warp * GV_ROWS * MP;

    for (int i = 0; have; ++i) {
        float yacc[NT][4];
        for (int s = it.s0; s < it.s1; ++s) {
            // one slab: up to 8 steps, chain = step parity; loads run NB steps ahead
            float c0[NT][4], c1[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) { c0[nt][q] = 0.f; c1[nt][q] = 0.f; }
            const int base = s * GV_SLAB_STEPS;
#pragma unroll
            for (int jj = 0; jj < GV_SLAB_STEPS; ++jj) {
                const int j = jj % NB;
                const int step = base + jj;
                if (step < steps_total) {
                    const uint4 a0 = A0[j], a1 = A1[j];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 Bv = lds128(xb + nt * 8 * XS + step * 32);
                        float (&acc)[4] = (jj & 1) ? c1[nt] : c0[nt];
                        mma_bf16_16816(acc, a0.x, a1.x, a0.y, a1.y, Bv.x, Bv.y);
                        mma_bf16_16816(acc, a0.z, a1.z, a0.w, a1.w, Bv.z, Bv.w);
                    }
                    // refill this register slot with the step NB ahead (same item)
                    const int nxt = step + NB;
                    if (nxt < it.s1 * GV_SLAB_STEPS) load_step(j, nxt);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float part = c0[nt][q] + c1[nt][q];
                    yacc[nt][q] = (p.split || s == 0) ? part : yacc[nt][q] + part;
                }
        }
        const int rb = it.rb, s_item = it.s0;
        // next item: start its loads before this item's epilogue
        GvItem nx;
        have = gv_item(p, slot, i + 1, &nx);
        if (have) {
            set_rows(nx.rb);
#pragma unroll
            for (int j = 0; j < NB; ++j) load_step(j, nx.s0 * GV_SLAB_STEPS + j);
        }
        gv_finish<NT, EPI>(p, rb, s_item, yacc, lane, cb, best);
        it = nx;
    }
    if (EPI == EPI_ARGMAX)
        gv_argmax_cta<NT>(p, best, amax_v, amax_i, warp, lane, tid, GV_CW, blockIdx.x, gridDim.x, false);
}

// Pack a row-major [rows][K] bf16 matrix into the fragment-ordered tiles.
// mode 0: plain (virtual row v = logical row v); mode 1 / 2: the gate / up half
// of a SwiGLU pair (tile rows 0..7 / 8..15 of row block rb are rows 8rb..8rb+7);
// mode 3: the attention in-projection in rope_src_row's order.
// One thread per 16-byte destination chunk; chunks of the other half are left
// untouched in modes 1 and 2; rows past the matrix are written as zero.
__global__ void k_pack_weight(const bf16_t* __restrict__ src, bf16_t* __restrict__ dst, int rows, int K,
                              int n_rowblk, int mode, int rope_nq, int rope_nkv, int rope_hd) {
    const int steps = K >> 5;
    const int64_t total = (int64_t)n_rowblk * steps * 64;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < total;
         q += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tile = q >> 6;
        const int within = (int)(q & 63), half = within >> 5, lane = within & 31;
        if ((mode == 1 && half) || (mode == 2 && !half)) continue;
        const int64_t rb = tile / steps;
        const int step = (int)(tile % steps);
        const int i = (lane >> 2) + 8 * half, c = lane & 3;
        const int64_t row = mode == 0 ? rb * 16 + i
                          : mode == 3 ? rope_src_row(rb * 16 + i, rope_nq, rope_nkv, rope_hd)
                                      : rb * 8 + (i & 7);
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < rows) v = *reinterpret_cast<const uint4*>(src + row * K + step * 32 + 8 * c);
        *reinterpret_cast<uint4*>(dst + gv_tile_elem(rb, step, steps, half, lane)) = v;
    }
}

// Plain copy of n bf16 values (small tensors of the weight arena).
__global__ void k_copy_u16(const bf16_t* __restrict__ src, bf16_t* __restrict__ dst, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = src[i];
}

// Reduce the per-CTA argmax partials of each row: the largest value, the lowest
// index among equal values; a NaN anywhere makes the row's argmax -1 and sets
// HGD_ERR_NAN.
__global__ void k_argmax_finalize(const float* __restrict__ best_v, const int32_t* __restrict__ best_i,
                                  int G, int M, int32_t* __restrict__ argmax, int32_t* status,
                                  int32_t* pos, int B, int T) {
    pdl_launch();
    pdl_wait();
    const int n = blockIdx.x;
    __shared__ float sv[32];
    __shared__ int si[32];
    __shared__ int snan;
    if (threadIdx.x == 0) snan = 0;
    __syncthreads();
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int i = best_i[n * G + g];
        const float v = best_v[n * G + g];
        if (i < 0) { snan = 1; continue; }
        if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
    }
    // warp then block reduction with the same comparator
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    const int wid = threadIdx.x >> 5, ln = threadIdx.x & 31;
    if (ln == 0) { sv[wid] = bv; si[wid] = bi; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (sv[w] > bv || (sv[w] == bv && si[w] < bi)) { bv = sv[w]; bi = si[w]; }
        if (snan) {
            argmax[n] = -1;
            set_status(status, HGD_ERR_NAN);
        } else {
            argmax[n] = bi;
        }
        if (pos && n == 0)
            for (int b = 0; b < B; ++b) pos[b] += T;
    }
}

}  // namespace hgd
