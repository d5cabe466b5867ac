// gemv.cuh -- weight-streaming BF16 GEMV / small-M GEMM engine for sm_100a.
//
// y[m][n] = sum_k x[m][k] W[n][k]  ("decode_linear_benchmark.md" commit message:
// BF16 GEMV and fused up/gate SwiGLU for decode shapes).  Design for B200:
//  * one producer warp streams 16-row weight tiles into a shared-memory ring with
//    1-D bulk copies (cp.async.bulk, one per row segment, mbarrier transaction
//    counts, L2 evict-first since weights are read once per step);
//  * eight consumer warps split each tile's k-block and run mma.sync m16n8k16
//    with the weight rows as the MMA M dimension and up to 32 tokens as N
//    (swap-AB), fp32 accumulation; rows are padded by 16 bytes in shared memory
//    so every 128-bit fragment load is bank-conflict free;
//  * the k-dimension is cut into equal blocks of <= 1024 (a function of K only);
//    each block's partial is reduced over the warps in a fixed order and the
//    block partials are added in block order, so every output's arithmetic
//    depends on K alone (not on M, N, the grid or the SM count);
//  * fused prologues (RMSNorm of the residual stream, embedding gather, gated
//    RMSNorm) and epilogues (fp32 / bf16 store, residual add, SwiGLU, argmax);
//  * programmatic dependent launch: weights stream before the previous kernel
//    in the stream has finished; activations are read after griddepcontrol.wait.
#pragma once

#include "common.cuh"

namespace hgd {

constexpr int GV_WARPS = 8;
constexpr int GV_THREADS = (GV_WARPS + 1) * 32;
constexpr int GV_ROWS = 16;
constexpr int GV_KB_MAX = 1024;
constexpr int GV_PAD = 8;  // bf16 elements of padding per shared-memory row
constexpr int GV_PITCH = 17;  // floats per token in the reduction buffers
constexpr int GV_SMEM_LIMIT = 227 * 1024;
constexpr int GV_MAX_STAGES = 8;

enum GvPrologue { PRO_COPY = 0, PRO_RMSNORM = 1, PRO_EMBED_RMSNORM = 2, PRO_GATED_NORM = 3 };
enum GvEpilogue { EPI_F32 = 0, EPI_BF16 = 1, EPI_RESID = 2, EPI_SWIGLU = 3, EPI_ARGMAX = 4 };

struct GemvParams {
    const bf16_t* W;   // [N][K]; SwiGLU: gate weights [I][K]
    const bf16_t* W2;  // SwiGLU: up weights [I][K]
    int N, K, M;       // N output features, M token rows of this launch
    int kb, nkb;       // k-block width (multiple of 32) and count
    int n_rowblk;      // row blocks (16 rows; SwiGLU: 8 gate + 8 up rows)
    int nstage, stage_bytes, x_bytes;
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
    int32_t* status;
};

__host__ __device__ inline int gv_align16(int v) { return (v + 15) & ~15; }

// Equal k-blocks of at most GV_KB_MAX, multiples of 32.  Depends on K only.
__host__ __device__ inline void gv_kblocks(int K, int* kb, int* nkb) {
    int n = (K + GV_KB_MAX - 1) / GV_KB_MAX;
    int w = (K + n - 1) / n;
    w = (w + 31) & ~31;
    *kb = w;
    *nkb = (K + w - 1) / w;
}

__device__ __forceinline__ bool bar_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Source row of tile row i (0..15) of row block rb; nullptr if past the end.
__device__ __forceinline__ const bf16_t* gv_row(const GemvParams& p, int EPI_SWI, int rb, int i) {
    if (EPI_SWI) {
        const int r = rb * 8 + (i & 7);
        if (r >= p.N) return nullptr;
        return (i < 8 ? p.W : p.W2) + (int64_t)r * p.K;
    }
    const int r = rb * GV_ROWS + i;
    if (r >= p.N) return nullptr;
    return p.W + (int64_t)r * p.K;
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
            float ss = 0.f;
            for (int c = lane; c < K / 8; c += 32) {
                const uint4 v = *reinterpret_cast<const uint4*>(src + c * 8);
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
                const uint4 v = *reinterpret_cast<const uint4*>(src + c * 8);
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
template <int NT, int PRO, int EPI>
__global__ void __launch_bounds__(GV_THREADS, 1) k_gemv(const __grid_constant__ GemvParams p) {
    constexpr int MP = 8 * NT;
    constexpr bool SWI = (EPI == EPI_SWIGLU);
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = p.K;
    const int XS = K + GV_PAD;           // elements per xs row
    const int RS = p.kb + GV_PAD;        // elements per stage row
    uint8_t* stages = smem;
    bf16_t* xs = reinterpret_cast<bf16_t*>(smem + p.nstage * p.stage_bytes);
    float* red = reinterpret_cast<float*>(smem + p.nstage * p.stage_bytes + p.x_bytes);
    float* yacc = red + GV_WARPS * MP * GV_PITCH;
    uint64_t* full = reinterpret_cast<uint64_t*>(yacc + MP * GV_PITCH + (MP * GV_PITCH & 1));
    uint64_t* empty = full + GV_MAX_STAGES;
    volatile int* abort_s = reinterpret_cast<volatile int*>(empty + GV_MAX_STAGES);

    if (tid == 0) {
        for (int s = 0; s < p.nstage; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GV_WARPS);
        }
        *abort_s = 0;
        mbar_fence_init();
    }
    __syncthreads();
    pdl_launch();

    // ------------------------------------------------------------ producer
    if (warp == GV_WARPS) {
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        int filled[GV_MAX_STAGES];
        for (int s = 0; s < GV_MAX_STAGES; ++s) filled[s] = -1;
        int it = 0;
        bool ok = true;
        for (int rb = blockIdx.x; ok && rb < p.n_rowblk; rb += gridDim.x) {
            for (int j = 0; j < p.nkb; ++j, ++it) {
                const int s = it % p.nstage;
                const uint32_t round = (uint32_t)(it / p.nstage);
                if (!mbar_wait_bounded(&empty[s], (round & 1) ^ 1, abort_s)) {
                    if (!*abort_s) set_status(p.status, HGD_ERR_TIMEOUT);
                    *abort_s = 1;
                    ok = false;
                    break;
                }
                const int k0 = j * p.kb;
                const int kbw = (j == p.nkb - 1) ? K - k0 : p.kb;
                const uint32_t rbytes = (uint32_t)kbw * 2u;
                uint32_t total = 0;
                for (int i = 0; i < GV_ROWS; ++i)
                    if (gv_row(p, SWI, rb, i)) total += rbytes;
                mbar_arrive_expect_tx(&full[s], total);
                uint8_t* dst = stages + s * p.stage_bytes;
                for (int i = 0; i < GV_ROWS; ++i) {
                    const bf16_t* src = gv_row(p, SWI, rb, i);
                    if (src) bulk_g2s(dst + i * RS * 2, src + k0, rbytes, &full[s], pol);
                }
                filled[s] = (int)(round & 1);
            }
        }
        // Do not leave while a copy into this CTA's shared memory is in flight.
        for (int s = 0; s < p.nstage; ++s)
            if (filled[s] >= 0) (void)mbar_wait_bounded(&full[s], (uint32_t)filled[s], nullptr);
        return;
    }

    // ----------------------------------------------------------- consumers
    const int ctid = tid;  // 0..255
    pdl_wait();
    gv_prologue<MP, PRO>(p, xs, ctid, warp, lane, yacc);
    named_bar(1, GV_WARPS * 32);

    const int r = lane >> 2, c = lane & 3;
    float best_v = -INFINITY;
    int best_i = 0x7fffffff;
    bool saw_nan = false;
    int it = 0;
    bool aborted = false;
    for (int rb = blockIdx.x; !aborted && rb < p.n_rowblk; rb += gridDim.x) {
        for (int j = 0; j < p.nkb; ++j, ++it) {
            const int s = it % p.nstage;
            const uint32_t round = (uint32_t)(it / p.nstage);
            const bool got = mbar_wait_bounded(&full[s], round & 1, abort_s);
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
            const int k0 = j * p.kb;
            const int kbw = (j == p.nkb - 1) ? K - k0 : p.kb;
            if (got) {
                const int S = kbw >> 5;
                const int s0 = (warp * S) / GV_WARPS, s1 = ((warp + 1) * S) / GV_WARPS;
                const bf16_t* tile = reinterpret_cast<const bf16_t*>(stages + s * p.stage_bytes);
                const bf16_t* a_lo = tile + r * RS + 8 * c;
                const bf16_t* a_hi = tile + (r + 8) * RS + 8 * c;
                const bf16_t* xb = xs + r * XS + k0 + 8 * c;
#pragma unroll 2
                for (int st = s0; st < s1; ++st) {
                    const uint4 A0 = lds128(a_lo + st * 32);
                    const uint4 A1 = lds128(a_hi + st * 32);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint4 Bv = lds128(xb + nt * 8 * XS + st * 32);
                        mma_bf16_16816(acc[nt], A0.x, A1.x, A0.y, A1.y, Bv.x, Bv.y);
                        mma_bf16_16816(acc[nt], A0.z, A1.z, A0.w, A1.w, Bv.z, Bv.w);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            } else if (!*abort_s) {
                set_status(p.status, HGD_ERR_TIMEOUT);
                *abort_s = 1;
            }
            // warp partials -> red[warp][token][row]
            float* rw = red + warp * MP * GV_PITCH;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int n0 = nt * 8 + 2 * c;
                rw[n0 * GV_PITCH + r] = acc[nt][0];
                rw[(n0 + 1) * GV_PITCH + r] = acc[nt][1];
                rw[n0 * GV_PITCH + r + 8] = acc[nt][2];
                rw[(n0 + 1) * GV_PITCH + r + 8] = acc[nt][3];
            }
            if (bar_or(1, GV_WARPS * 32, !got || *abort_s)) {
                aborted = true;
                break;
            }
            // fixed-order reduction over warps, then over k-blocks
            for (int e = ctid; e < MP * GV_ROWS; e += GV_WARPS * 32) {
                const int n = e >> 4, i = e & 15;
                float sum = red[n * GV_PITCH + i];
#pragma unroll
                for (int w = 1; w < GV_WARPS; ++w) sum += red[w * MP * GV_PITCH + n * GV_PITCH + i];
                yacc[n * GV_PITCH + i] = (j == 0) ? sum : yacc[n * GV_PITCH + i] + sum;
            }
            named_bar(1, GV_WARPS * 32);
            if (j != p.nkb - 1) continue;

            // ----------------------------------------------------- epilogue
            if (EPI == EPI_SWIGLU) {
                for (int e = ctid; e < MP * 8; e += GV_WARPS * 32) {
                    const int n = e >> 3, i = e & 7;
                    const int col = rb * 8 + i;
                    if (n < p.M && col < p.N) {
                        const float g = yacc[n * GV_PITCH + i], u = yacc[n * GV_PITCH + i + 8];
                        reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(silu_f(g) * u);
                    }
                }
            } else if (EPI == EPI_ARGMAX) {
                for (int e = ctid; e < MP * GV_ROWS; e += GV_WARPS * 32) {
                    const int n = e >> 4, i = e & 15;
                    const int col = rb * GV_ROWS + i;
                    if (p.logits && n < p.M && col < p.N) p.logits[n * p.logits_ld + col] = yacc[n * GV_PITCH + i];
                }
                if (ctid < p.M) {
                    const int n = ctid;
                    for (int i = 0; i < GV_ROWS; ++i) {
                        const int col = rb * GV_ROWS + i;
                        if (col >= p.N) break;
                        const float v = yacc[n * GV_PITCH + i];
                        if (v != v) saw_nan = true;
                        else if (v > best_v || (v == best_v && col < best_i)) { best_v = v; best_i = col; }
                    }
                }
            } else {
                for (int e = ctid; e < MP * GV_ROWS; e += GV_WARPS * 32) {
                    const int n = e >> 4, i = e & 15;
                    const int col = rb * GV_ROWS + i;
                    if (n >= p.M || col >= p.N) continue;
                    const float v = yacc[n * GV_PITCH + i];
                    if (EPI == EPI_F32) {
                        reinterpret_cast<float*>(p.y)[n * p.y_ld + col] = v;
                    } else if (EPI == EPI_BF16) {
                        reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(v);
                    } else {  // EPI_RESID: y = bf16(resid + v)
                        const float base = bf2f(p.resid[n * p.resid_ld + col]);
                        reinterpret_cast<bf16_t*>(p.y)[n * p.y_ld + col] = f2bf(base + v);
                    }
                }
            }
        }
    }
    if (EPI == EPI_ARGMAX && ctid < p.M) {
        p.best_v[ctid * gridDim.x + blockIdx.x] = best_v;
        p.best_i[ctid * gridDim.x + blockIdx.x] = saw_nan ? -1 : best_i;
    }
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
