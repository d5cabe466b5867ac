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
