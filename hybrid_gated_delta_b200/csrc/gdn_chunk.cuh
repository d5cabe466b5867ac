// gdn_chunk.cuh -- the gated delta rule over many rows at once (prefill).
//
// "luce-megakernel HANDOFF.md", Architecture Summary (a prefill kernel beside
// the decode kernel) and Expected Results (pp512).  A prompt of T rows gives the
// same state and outputs as T one-row steps of the gated delta rule
//   S_t = alpha_t S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - alpha_t S_{t-1} k_t),
//   o_t = S_t q_t,
// but the rows of a chunk of C are taken together.  With Gamma_t the product of
// alpha over the chunk's rows up to t (G_t its logarithm, the running sum of g)
// and S_0 the state before the chunk, unrolling the recurrence gives
//   (I + A) U = diag(beta) (V - diag(Gamma) K S_0^T),
//       A[t][s] = beta_t exp(G_t - G_s) (k_s . k_t)   for s < t   (unit lower triangular system)
//   o_t = Gamma_t S_0 q_t + sum_{s <= t} exp(G_t - G_s) (q_t . k_s) u_s
//   S_C = Gamma_C S_0 + sum_s exp(G_C - G_s) u_s k_s^T
// (rows of U are the rows' writes u_t).  Every product above is separable over
// the value rows of the state, so a CTA owns GCK_DVB value rows of one (stream,
// head) and runs the chunks of the prompt in order; the small C x C matrices are
// formed redundantly by the CTAs of a head.  fp32 throughout, on the CUDA cores:
// bf16 or tf32 tensor-core products would not keep the state within its 1e-4
// tolerance.  The state sits in shared memory transposed (key element major), so
// the products read it without bank conflicts; the triangular solve runs in
// registers, one lane per value row.  Results equal the one-row steps to fp32
// rounding, not bit for bit (the sums are ordered differently).
#pragma once

#include "gdn.cuh"

namespace hgd {

constexpr int GCK_C = 32;        // rows per chunk
constexpr int GCK_DVB = 32;      // value rows of the state per CTA
constexpr int GCK_THREADS = 256;

struct GdnChunkParams {
    const float* q; const float* k; const float* v; int64_t stride;  // rows (b*T + t), as hgd_gdn_decode_step
    const float* g; const float* b;                                   // [B*T][H] raw
    float* S;                                                         // [B][H][dv][dk], in place
    float* o;                                                         // [B][T][H][dv]
    int B, T, H, dv, l2norm;
};

template <int DK>
struct GckSmem {
    static constexpr int KS = DK + 4;  // row stride of q and k (16-byte aligned, spreads the lanes' rows)
    float st[DK * GCK_DVB];            // the state slice, transposed: st[j][i] = S[i0 + i][j]
    float qs[GCK_C * KS], ks[GCK_C * KS];
    float vs[GCK_C * GCK_DVB];         // the chunk's values of this slice; then the writes U
    float xs[GCK_C * GCK_DVB];         // K S_0^T, then Q S_0^T
    float A[GCK_C * GCK_C], P[GCK_C * GCK_C];
    float G[GCK_C], beta[GCK_C];
};

// grid (B * H, dv / GCK_DVB), block 256.
template <int DK>
__global__ void __launch_bounds__(GCK_THREADS, 2) k_gdn_chunked(const __grid_constant__ GdnChunkParams p) {
    pdl_launch();
    pdl_wait();
    extern __shared__ __align__(16) uint8_t gck_raw[];
    GckSmem<DK>& sm = *reinterpret_cast<GckSmem<DK>*>(gck_raw);
    constexpr int KS = GckSmem<DK>::KS, C = GCK_C, DVB = GCK_DVB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H, i0 = blockIdx.y * DVB;
    float* Sg = p.S + ((int64_t)(b * p.H + h) * p.dv + i0) * DK;

    // the state slice, transposed
    for (int e = tid; e < DVB * DK; e += GCK_THREADS) {
        const int i = e / DK, j = e % DK;
        sm.st[j * DVB + i] = Sg[(int64_t)i * DK + j];
    }

    for (int t0 = 0; t0 < p.T; t0 += C) {
        const int c = min(C, p.T - t0);
        __syncthreads();  // the previous chunk is done with every buffer
        // the chunk's rows; rows past the prompt are zero with g = 0, beta = 0 (no effect)
        for (int e = tid; e < C * (DK / 4); e += GCK_THREADS) {
            const int t = e / (DK / 4), j = (e % (DK / 4)) * 4;
            float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), kv = qv;
            if (t < c) {
                const int64_t row = (int64_t)b * p.T + t0 + t;
                qv = *reinterpret_cast<const float4*>(p.q + row * p.stride + (int64_t)h * DK + j);
                kv = *reinterpret_cast<const float4*>(p.k + row * p.stride + (int64_t)h * DK + j);
            }
            *reinterpret_cast<float4*>(&sm.qs[t * KS + j]) = qv;
            *reinterpret_cast<float4*>(&sm.ks[t * KS + j]) = kv;
        }
        for (int e = tid; e < C * DVB; e += GCK_THREADS) {
            const int t = e / DVB, i = e % DVB;
            sm.vs[e] = t < c ? p.v[((int64_t)b * p.T + t0 + t) * p.stride + (int64_t)h * p.dv + i0 + i] : 0.f;
        }
        if (warp == 0) {
            // G_t = running sum of g over the chunk (inclusive scan), beta_t
            float gt = 0.f, bt = 0.f;
            if (lane < c) {
                const int64_t row = (int64_t)b * p.T + t0 + lane;
                gt = p.g[row * p.H + h];
                bt = sigmoid_f(p.b[row * p.H + h]);
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, gt, o);
                if (lane >= o) gt += u;
            }
            sm.G[lane] = gt;
            sm.beta[lane] = bt;
        }
        __syncthreads();
        // L2 normalisation of the q and k rows: x / sqrt(sum x^2 + 1e-6), warp w rows w, w + 8, ...
        if (p.l2norm) {
            for (int t = warp; t < C; t += GCK_THREADS / 32) {
#pragma unroll
                for (int which = 0; which < 2; ++which) {
                    float* r = (which ? sm.ks : sm.qs) + t * KS;
                    float ss = 0.f;
                    for (int j = lane; j < DK; j += 32) ss = fmaf(r[j], r[j], ss);
                    const float sc = rsqrtf(warp_sum(ss) + 1e-6f);
                    for (int j = lane; j < DK; j += 32) r[j] = r[j] * sc;
                }
            }
            __syncthreads();
        }
        // A (strictly lower: beta_t e^(G_t - G_s) k_s.k_t) and P (lower with the
        // diagonal: e^(G_t - G_s) q_t.k_s): lane s, rows t = warp + 8m
        {
            const int s = lane;
            float dA[4], dP[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) { dA[m] = 0.f; dP[m] = 0.f; }
            for (int j = 0; j < DK; j += 4) {
                const float4 kv = *reinterpret_cast<const float4*>(&sm.ks[s * KS + j]);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int t = warp + 8 * m;
                    const float4 kt = *reinterpret_cast<const float4*>(&sm.ks[t * KS + j]);
                    const float4 qt = *reinterpret_cast<const float4*>(&sm.qs[t * KS + j]);
                    dA[m] = fmaf(kt.x, kv.x, fmaf(kt.y, kv.y, fmaf(kt.z, kv.z, fmaf(kt.w, kv.w, dA[m]))));
                    dP[m] = fmaf(qt.x, kv.x, fmaf(qt.y, kv.y, fmaf(qt.z, kv.z, fmaf(qt.w, kv.w, dP[m]))));
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int t = warp + 8 * m;
                const float dec = s <= t ? expf(sm.G[t] - sm.G[s]) : 0.f;
                sm.A[t * C + s] = s < t ? sm.beta[t] * dec * dA[m] : 0.f;
                sm.P[t * C + s] = dec * dP[m];
            }
        }
        // X = K S_0^T and Y = Q S_0^T on this slice: lane i, rows t = warp + 8m
        float yq[4];
        {
            float xk[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) { xk[m] = 0.f; yq[m] = 0.f; }
            for (int j = 0; j < DK; j += 4) {
                const float s0 = sm.st[(j + 0) * DVB + lane], s1 = sm.st[(j + 1) * DVB + lane];
                const float s2 = sm.st[(j + 2) * DVB + lane], s3 = sm.st[(j + 3) * DVB + lane];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int t = warp + 8 * m;
                    const float4 kt = *reinterpret_cast<const float4*>(&sm.ks[t * KS + j]);
                    const float4 qt = *reinterpret_cast<const float4*>(&sm.qs[t * KS + j]);
                    xk[m] = fmaf(kt.x, s0, fmaf(kt.y, s1, fmaf(kt.z, s2, fmaf(kt.w, s3, xk[m]))));
                    yq[m] = fmaf(qt.x, s0, fmaf(qt.y, s1, fmaf(qt.z, s2, fmaf(qt.w, s3, yq[m]))));
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) sm.xs[(warp + 8 * m) * DVB + lane] = xk[m];
        }
        __syncthreads();
        // the writes: (I + A) U = diag(beta) (V - diag(Gamma) X), forward substitution
        // down the chunk, one lane per value row (warp 0); U replaces V
        if (warp == 0) {
            float u[C];
#pragma unroll
            for (int t = 0; t < C; ++t) {
                float r = sm.beta[t] * (sm.vs[t * DVB + lane] - expf(sm.G[t]) * sm.xs[t * DVB + lane]);
#pragma unroll
                for (int s = 0; s < t; ++s) r = fmaf(-sm.A[t * C + s], u[s], r);
                u[t] = r;
                sm.vs[t * DVB + lane] = r;
            }
        }
        __syncthreads();
        // o_t = Gamma_t (Q S_0^T)[t] + sum_{s <= t} P[t][s] u_s
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int t = warp + 8 * m;
            float acc = expf(sm.G[t]) * yq[m];
            for (int s = 0; s <= t; ++s) acc = fmaf(sm.P[t * C + s], sm.vs[s * DVB + lane], acc);
            if (t < c)
                p.o[(((int64_t)b * p.T + t0 + t) * p.H + h) * p.dv + i0 + lane] = acc;
        }
        // S_C = Gamma_C S_0 + sum_s e^(G_C - G_s) u_s k_s^T on the slice: lane i, key
        // elements j = 16 warp .. 16 warp + 15 (rows past the prompt add nothing)
        {
            const float gc = sm.G[C - 1];
            const float ec = expf(gc);
            float acc[DK / 8];
#pragma unroll
            for (int jj = 0; jj < DK / 8; ++jj) acc[jj] = ec * sm.st[(warp * (DK / 8) + jj) * DVB + lane];
            for (int s = 0; s < C; ++s) {
                const float us = expf(gc - sm.G[s]) * sm.vs[s * DVB + lane];
#pragma unroll
                for (int jj = 0; jj < DK / 8; ++jj) acc[jj] = fmaf(us, sm.ks[s * KS + warp * (DK / 8) + jj], acc[jj]);
            }
            __syncthreads();  // every thread is done reading the old state
#pragma unroll
            for (int jj = 0; jj < DK / 8; ++jj) sm.st[(warp * (DK / 8) + jj) * DVB + lane] = acc[jj];
        }
    }
    __syncthreads();
    for (int e = tid; e < DVB * DK; e += GCK_THREADS) {
        const int i = e / DK, j = e % DK;
        Sg[(int64_t)i * DK + j] = sm.st[j * DVB + i];
    }
}

}  // namespace hgd
