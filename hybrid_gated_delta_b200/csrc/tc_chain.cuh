// tc_chain.cuh -- the per-row kernels of the tensor-core decode chain.
//
// "qwen3_5 cuda: mixed-width MLX checkpoints ... #849", PR body: windows of rows
// (several streams of up to 16 rows each) whose rows equal one-row steps bit for
// bit.  In the tensor-core chain every projection is one tcgen05 GEMM
// (gemm_tc.cuh) over all of a call's token rows, and the tensor cores give each
// token row the same result whatever the number of rows the call carries; the
// kernels here are the work between the GEMMs, each computing every row from
// that row's inputs alone.  So a window through this chain equals its one-row
// steps through it, bit for bit, as the mma.sync chain's windows equal its
// steps.  (The two chains sum their dot products in different orders: their
// results agree to fp32 rounding, not bit for bit.)
#pragma once

#include "attn.cuh"
#include "gemv.cuh"

namespace hgd {

// Causal conv over the first C columns of the in-projection rows, in place: one
// thread per (stream, channel), rows in order, as k_conv_tail (tail records per
// row when tail_rec is set).  Row (b, t) is x + (b*T + t) * x_ld.
struct TcConvParams {
    float* x; int64_t x_ld; float* tail; const bf16_t* w; float* tail_rec;
    int B, T, C;
};
// REC: tail records on (tail_rec set).  Each thread stages its channel's inputs
// of up to 16 rows in shared memory at once (cp.async; every thread reads back
// only its own column, so no barrier), then runs the rows in order.
template <bool REC>
__global__ void __launch_bounds__(256) k_tc_conv(const __grid_constant__ TcConvParams p) {
    constexpr int RB = 16;
    __shared__ float xs[RB][256];
    pdl_launch();
    pdl_wait();
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)p.B * p.C) return;
    const int b = (int)(idx / p.C), c = (int)(idx % p.C), tid = threadIdx.x;
    constexpr int NT = GV_CONV_K - 1;
    float tl[NT], w[GV_CONV_K];
#pragma unroll
    for (int j = 0; j < GV_CONV_K; ++j) w[j] = bf2f(p.w[(int64_t)c * GV_CONV_K + j]);
    float* tb = p.tail + (int64_t)b * NT * p.C + c;
#pragma unroll
    for (int j = 0; j < NT; ++j) tl[j] = tb[(int64_t)j * p.C];
    const int64_t ld = p.x_ld;
    float* xb = p.x + (int64_t)b * p.T * ld + c;  // row t of this stream at xb + t * ld
    for (int t0 = 0; t0 < p.T; t0 += RB) {
        const int n = min(RB, p.T - t0);
        for (int u = 0; u < n; ++u) cp_async4(&xs[u][tid], xb + (int64_t)(t0 + u) * ld);
        cp_async_commit();
        cp_async_wait_all();
        for (int u = 0; u < n; ++u) {
            const int t = t0 + u;
            const float xv = xs[u][tid];
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < NT; ++j) acc = fmaf(w[j], tl[j], acc);
            acc = fmaf(w[NT], xv, acc);
            xb[(int64_t)t * ld] = silu_f(acc);
#pragma unroll
            for (int j = 0; j + 1 < NT; ++j) tl[j] = tl[j + 1];
            tl[NT - 1] = xv;
            if (REC) {
                float* rp = p.tail_rec + ((int64_t)b * p.T + t) * NT * p.C + c;
#pragma unroll
                for (int j = 0; j < NT; ++j) rp[(int64_t)j * p.C] = tl[j];
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) tb[(int64_t)j * p.C] = tl[j];
}

// RoPE of the query and key heads of each row and the append of its key and
// value rows to the cache at position pos[b] + t (rotate-half pairs (i, i +
// hd/2), base^(-2i/hd) angles as the mma.sync chain's epilogue computes them).
// In-projection rows, logical order: q (nq*hd) | gate (nq*hd) | k (nkv*hd) |
// v (nkv*hd) at y + m * y_ld.  One CTA per token row.
struct TcRopeParams {
    const float* y; int64_t y_ld;
    float* qrot;                     // [M][nq*hd]
    bf16_t* kcache; bf16_t* vcache;  // this layer: [B][nkv][Lmax][hd]
    const int32_t* pos; int32_t* status;
    int T, nq, nkv, hd, Lmax;
    double inv1;
};
__global__ void k_tc_rope(const __grid_constant__ TcRopeParams p) {
    pdl_launch();
    pdl_wait();
    const int m = blockIdx.x, b = m / p.T, t = m % p.T;
    const int P = p.pos[b] + t, hd = p.hd, half = hd / 2;
    const float* yr = p.y + (int64_t)m * p.y_ld;
    if (P < 0 || P >= p.Lmax) {
        if (threadIdx.x == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
        return;
    }
    // the row's angles, one per rotated pair, shared by every head (rope_sincos at P)
    __shared__ float rsn[ATTN_MAX_HD / 2], rcs[ATTN_MAX_HD / 2];
    for (int i = threadIdx.x; i < half; i += blockDim.x) rope_sincos(P, i, p.inv1, &rsn[i], &rcs[i]);
    __syncthreads();
    const int nqp = p.nq * half, nkp = p.nkv * half;
    for (int e = threadIdx.x; e < nqp + nkp + p.nkv * hd; e += blockDim.x) {
        if (e < nqp + nkp) {
            const bool isk = e >= nqp;
            const int ee = isk ? e - nqp : e, head = ee / half, i = ee % half;
            const float* src = yr + (isk ? 2 * (int64_t)p.nq * hd : 0) + (int64_t)head * hd;
            const float a = src[i], bb = src[i + half];
            const float sn = rsn[i], cs = rcs[i];
            const float x0 = a * cs - bb * sn, x1 = bb * cs + a * sn;
            if (!isk) {
                float* qo = p.qrot + (int64_t)m * p.nq * hd + (int64_t)head * hd;
                qo[i] = x0;
                qo[i + half] = x1;
            } else {
                bf16_t* ko = p.kcache + (((int64_t)b * p.nkv + head) * p.Lmax + P) * hd;
                ko[i] = f2bf(x0);
                ko[i + half] = f2bf(x1);
            }
        } else {
            const int ev = e - nqp - nkp, g = ev / hd, d = ev % hd;
            p.vcache[(((int64_t)b * p.nkv + g) * p.Lmax + P) * hd + d] =
                f2bf(yr[2 * (int64_t)p.nq * hd + (int64_t)p.nkv * hd + (int64_t)g * hd + d]);
        }
    }
}

// ---------------------------------------------------------------- attention partials on the tensor cores
// The attention partials of the window's (row, query head) vectors: with every
// row of a stream at once, the scores of a chunk are the dense product of the
// stream's query vectors and the chunk's keys, and the weighted values the
// product of the weights and the chunk's value rows ("qwen3_5 cuda: mixed-width
// MLX checkpoints ... #849", PR body: gated attention, chunk partials and a
// merge, a window's rows summed exactly as their one-row steps).
// grid (B, nkv, max_chunks), block 256: one CTA per (stream, kv head, chunk of
// ATTN_CHUNK keys), as k_attn_partial, with the stream's vectors that reach the
// chunk as the rows of two mma.sync products, up to 64 vectors a pass:
//   S = Q K^T (vectors x the chunk's keys, over the head's dims: two partial
//             products over its two halves, summed first half first),
//   O = P V   (vectors x dims, over the chunk's keys).
// An fp32 operand enters as two bf16 terms, hi = bf16(x) and lo = bf16(x - hi)
// (the difference exact in fp32; hi + lo carries about 16 significant bits of x),
// against the bf16 cache rows, summed in fp32.  Per vector: s_j = S_j / sqrt(hd), m = max over the keys
// it sees, p_j = exp(s_j - m) for those and 0 for the rest, l = sum_j p_j
// (warp_sum), acc = O: the partial row (m, l, acc) k_attn_merge reads.
// A tensor-core output element depends on its own row and column only, the keys
// a vector does not see enter with p = 0 (a row beyond the chunk's last key is
// zero) and a zero result is stored as +0, so each vector's partial is the same
// whatever the number of rows in the call.
constexpr int ATTN_TC_V = 64;  // vectors a pass: four 16-row tiles
__host__ __device__ constexpr int attn_tc_row(int hd) { return hd + 8; }  // padded smem row (bf16)
__host__ __device__ inline size_t attn_tc_smem_bytes(int hd) {
    return (size_t)2 * ATTN_CHUNK * attn_tc_row(hd) * 2 + (size_t)2 * ATTN_TC_V * (ATTN_CHUNK + 1) * 4 +
           (size_t)2 * ATTN_TC_V * (ATTN_CHUNK + 8) * 2;
}

__device__ __forceinline__ void split_bf16x2(float2 x, uint32_t& hi, uint32_t& lo) {
    const bf16_t h0 = f2bf(x.x), h1 = f2bf(x.y);
    hi = (uint32_t)h0 | ((uint32_t)h1 << 16);
    lo = pack_bf2(x.x - bf2f(h0), x.y - bf2f(h1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}

// Warp (tile mt, half) of a pass: S over the dims [half HD/2, (half + 1) HD/2) of
// the tile's 16 vectors (the two halves summed afterwards, half 0 first), O over
// the same half of the dims.  Its query fragments (hi and lo terms of every
// 16-dim step of its half) are loaded into registers at once, before the wait
// for the chunk's rows.
template <int HD>
__global__ void __launch_bounds__(256, 2) k_attn_partial_tc(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(16) uint8_t attn_tc_smem[];
    constexpr int KS = attn_tc_row(HD), SS = ATTN_CHUNK + 1, PS = ATTN_CHUNK + 8;
    constexpr int KH = HD / 2, KST = KH / 16;  // a warp's dims, its 16-dim steps
    bf16_t* Ks = reinterpret_cast<bf16_t*>(attn_tc_smem);  // [ATTN_CHUNK][KS]
    bf16_t* Vs = Ks + ATTN_CHUNK * KS;
    float* Sm = reinterpret_cast<float*>(Vs + ATTN_CHUNK * KS);  // [2 halves][ATTN_TC_V][SS]
    bf16_t* Ph = reinterpret_cast<bf16_t*>(Sm + 2 * ATTN_TC_V * SS);  // [ATTN_TC_V][PS], hi and lo terms
    bf16_t* Pl = Ph + ATTN_TC_V * PS;
    pdl_launch();
    pdl_wait();
    const int b = blockIdx.x, g = blockIdx.y, ch = blockIdx.z;
    const int key0 = ch * ATTN_CHUNK, pos = p.pos[b];
    // the rows of this stream with a valid position that reaches the chunk
    int tlo = max(0, key0 - pos), thi = min(p.T, p.Lmax - pos);
    if (pos < 0) tlo = max(tlo, -pos);
    if (tlo >= thi) return;
    const int nkc = min(ATTN_CHUNK, pos + thi - key0);  // keys the chunk's last row sees
    const int64_t cache0 = (((int64_t)b * p.nkv + g) * p.Lmax + key0) * HD;
    // the chunk's key and value rows (cp.async, all in flight at once), zero beyond nkc
    constexpr int R16 = HD / 8;
    for (int i = threadIdx.x; i < ATTN_CHUNK * R16; i += blockDim.x) {
        const int r = i / R16, c = i % R16;
        bf16_t* kd = Ks + r * KS + c * 8;
        bf16_t* vd = Vs + r * KS + c * 8;
        if (r < nkc) {
            cp_async16(kd, p.kcache + cache0 + (int64_t)r * HD + c * 8);
            cp_async16(vd, p.vcache + cache0 + (int64_t)r * HD + c * 8);
        } else {
            *reinterpret_cast<uint4*>(kd) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(vd) = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    cp_async_commit();
    const int group = p.nq / p.nkv, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, cq = lane & 3;
    const int nv = (thi - tlo) * group;
    const float scale = 1.0f / sqrtf((float)HD);
    // vector v: row tlo + v / group of the stream, query head g * group + v % group
    auto vec_row = [&](int v) { return b * p.T + tlo + v / group; };
    auto vec_head = [&](int v) { return g * group + v % group; };
    auto part_of = [&](int v) {
        return p.part + (((int64_t)vec_row(v) * p.nq + vec_head(v)) * p.max_chunks + ch) * (HD + 2);
    };
    const int mt = warp & 3, half = warp >> 2;
    // A fragments of the tile at m0, this warp's dims: qa[k][0..3] hi, [4..7] lo,
    // registers (row gq, dims 2cq..), (gq + 8, 2cq..), (gq, 2cq + 8..), (gq + 8, 2cq + 8..)
    uint32_t qa[KST][8];
    auto load_q = [&](int m0) {
        const float* qr[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int v = m0 + gq + 8 * r;
            qr[r] = v < nv ? p.qrot + ((int64_t)vec_row(v) * p.nq + vec_head(v)) * HD + half * KH : nullptr;
        }
        float2 x[KST][4];
#pragma unroll
        for (int k = 0; k < KST; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float* q = qr[i & 1];
                x[k][i] = q ? *reinterpret_cast<const float2*>(q + 16 * k + 2 * cq + 8 * (i >> 1)) : make_float2(0.f, 0.f);
            }
#pragma unroll
        for (int k = 0; k < KST; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) split_bf16x2(x[k][i], qa[k][i], qa[k][4 + i]);
    };
    if (mt * 16 < nv) load_q(mt * 16);
    cp_async_wait_all();
    __syncthreads();
    for (int v0 = 0; v0 < nv; v0 += ATTN_TC_V) {
        const int m0 = v0 + mt * 16;
        if (m0 < nv) {
            if (v0 > 0) load_q(m0);
            float acc[4][4] = {};
#pragma unroll
            for (int k = 0; k < KST; ++k)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const bf16_t* kr = Ks + (8 * nt + gq) * KS + half * KH + 16 * k + 2 * cq;
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + 8);
                    mma_bf16_16816(acc[nt], qa[k][0], qa[k][1], qa[k][2], qa[k][3], b0, b1);
                    mma_bf16_16816(acc[nt], qa[k][4], qa[k][5], qa[k][6], qa[k][7], b0, b1);
                }
            float* sh = Sm + half * ATTN_TC_V * SS + (mt * 16 + gq) * SS;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int key = 8 * nt + 2 * cq;
                sh[key] = acc[nt][0];
                sh[key + 1] = acc[nt][1];
                sh[8 * SS + key] = acc[nt][2];
                sh[8 * SS + key + 1] = acc[nt][3];
            }
        }
        __syncthreads();
        // per vector (one warp, lane = key): s, m, p = exp(s - m) as hi and lo terms, l
        for (int vi = warp; vi < ATTN_TC_V; vi += 8) {
            const int v = v0 + vi;
            float e = 0.f;
            if (v < nv) {
                const int nk = min(ATTN_CHUNK, pos + tlo + v / group + 1 - key0);
                const float s = lane < nk ? (Sm[vi * SS + lane] + Sm[(ATTN_TC_V + vi) * SS + lane]) * scale : -INFINITY;
                float m = s;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                e = lane < nk ? expf(s - m) : 0.f;
                const float l = warp_sum(e);
                if (lane == 0) {
                    float* dst = part_of(v);
                    dst[0] = m;
                    dst[1] = l;
                }
            }
            const bf16_t eh = f2bf(e);
            Ph[vi * PS + lane] = eh;
            Pl[vi * PS + lane] = f2bf(e - bf2f(eh));
        }
        __syncthreads();
        if (m0 < nv) {
            uint32_t ph[2][4], pl[2][4];  // A: the tile's weights, keys 16 ks ..
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int o = (mt * 16 + gq) * PS + 16 * ks + 2 * cq;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int oi = o + 8 * PS * (i & 1) + 8 * (i >> 1);
                    ph[ks][i] = *reinterpret_cast<const uint32_t*>(Ph + oi);
                    pl[ks][i] = *reinterpret_cast<const uint32_t*>(Pl + oi);
                }
            }
            // B: value rows transposed by ldmatrix, two 8-dim tiles per load:
            // lane j * 8 + r addresses key 16 ks + r + 8 (j & 1), dim n0 + 8 (j >> 1)
            const int lj = lane >> 3, lr = lane & 7;
            float* dst[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int v = m0 + gq + 8 * r;
                dst[r] = v < nv ? part_of(v) + 2 : nullptr;
            }
            for (int n0 = half * KH; n0 < half * KH + KH; n0 += 16) {
                uint32_t bq[2][4];
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    ldsm_x4_trans(bq[ks], Vs + (16 * ks + lr + 8 * (lj & 1)) * KS + n0 + 8 * (lj >> 1));
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int ks = 0; ks < 2; ++ks) {
                        mma_bf16_16816(o, ph[ks][0], ph[ks][1], ph[ks][2], ph[ks][3], bq[ks][2 * nt], bq[ks][2 * nt + 1]);
                        mma_bf16_16816(o, pl[ks][0], pl[ks][1], pl[ks][2], pl[ks][3], bq[ks][2 * nt], bq[ks][2 * nt + 1]);
                    }
                    const int d = n0 + 8 * nt + 2 * cq;
#pragma unroll
                    for (int r = 0; r < 2; ++r)
                        if (dst[r]) *reinterpret_cast<float2*>(dst[r] + d) = make_float2(o[2 * r] + 0.f, o[2 * r + 1] + 0.f);
                }
            }
        }
        __syncthreads();  // the next pass rewrites S and P
    }
}

// argmax[m] over the fp32 logits row m (first maximum: lowest index on ties; a
// NaN gives -1 and HGD_ERR_NAN), in two passes.  k_tc_argmax_part: grid (M,
// TC_AM_SLICES), block 256; CTA (m, s) scans slice s of the row (contiguous
// index ranges, four loads in flight per thread) into the partial pv/pi[m][s]
// (pi = -2: the slice holds a NaN).  k_tc_argmax_final: grid M, one warp; the
// slices merge in index order; then, if pos is set, every stream's position
// advances by T (block 0).
constexpr int TC_AM_SLICES = 32;
__global__ void __launch_bounds__(256) k_tc_argmax_part(const float* logits, int64_t ld, int V, float* pv, int* pi) {
    pdl_launch();
    pdl_wait();
    const int m = blockIdx.x, sl = blockIdx.y;
    const int span = (V + TC_AM_SLICES - 1) / TC_AM_SLICES;
    const int lo = sl * span, hi = min(V, lo + span);
    const float* lr = logits + (int64_t)m * ld;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    bool nan = false;
    auto take = [&](float v, int i) {
        if (v != v) nan = true;
        else if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
    };
    int lo4 = lo;  // the 16-byte aligned part of the slice runs as float4 loads
    if ((ld & 3) == 0 && (lo & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15) == 0) {
        const int n4 = (hi - lo) / 4;
        const float4* l4 = reinterpret_cast<const float4*>(lr + lo);
        for (int q0 = (int)threadIdx.x; q0 < n4; q0 += 2 * 256) {
            float4 v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) v[u] = q0 + u * 256 < n4 ? l4[q0 + u * 256] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (q0 + u * 256 < n4) {
                    const int i = lo + 4 * (q0 + u * 256);
                    take(v[u].x, i); take(v[u].y, i + 1); take(v[u].z, i + 2); take(v[u].w, i + 3);
                }
        }
        lo4 = lo + 4 * n4;
    }
    constexpr int U = 4;
    for (int i0 = lo4 + (int)threadIdx.x; i0 < hi; i0 += U * 256) {
        float v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = i0 + u * 256 < hi ? lr[i0 + u * 256] : -INFINITY;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = i0 + u * 256;
            if (i >= hi) break;
            if (v[u] != v[u]) nan = true;
            else if (v[u] > bv || (v[u] == bv && i < bi)) { bv = v[u]; bi = i; }
        }
    }
    __shared__ float sv[8];
    __shared__ int si[8], sn[8];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    nan = __any_sync(0xffffffffu, nan);
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { sv[w] = bv; si[w] = bi; sn[w] = nan; }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool anynan = sn[0];
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k) {
            anynan = anynan || sn[k];
            if (sv[k] > bv || (sv[k] == bv && si[k] < bi)) { bv = sv[k]; bi = si[k]; }
        }
        pv[m * TC_AM_SLICES + sl] = bv;
        pi[m * TC_AM_SLICES + sl] = anynan ? -2 : bi;
    }
}
__global__ void k_tc_argmax_final(const float* pv, const int* pi, int32_t* argmax, int32_t* status, int32_t* pos,
                                  int B, int T) {
    pdl_launch();
    pdl_wait();
    const int m = blockIdx.x, lane = threadIdx.x;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    bool nan = false;
    if (lane < TC_AM_SLICES) {
        bv = pv[m * TC_AM_SLICES + lane];
        bi = pi[m * TC_AM_SLICES + lane];
        nan = bi == -2;
        if (nan) { bv = -INFINITY; bi = 0x7fffffff; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    nan = __any_sync(0xffffffffu, nan);
    if (lane == 0) {
        argmax[m] = nan ? -1 : bi;
        if (nan) set_status(status, HGD_ERR_NAN);
        if (pos && m == 0)
            for (int s = 0; s < B; ++s) pos[s] += T;
    }
}

}  // namespace hgd
