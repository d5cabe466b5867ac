// attn.cuh -- decode attention of the gated full-attention layers.
//
// "qwen3_5 cuda: mixed-width MLX checkpoints ... #849", PR body: gated attention
// with more query heads than key/value heads; partials over fixed-width key
// chunks plus a merge kernel with fp32 sums, the chunks cut at each key's
// logical position so that a row of a window sums exactly as its one-row step.
//
// Per row (stream b, window row t) at position P = pos[b] + t:
//   k_rope_append:   rotate-half RoPE of q and k at P (angles in double, then
//                    fp32), K and V written to the cache at P as bf16;
//   k_attn_partial:  per (row, kv head, chunk of CHUNK keys), the four query
//                    heads of the group: s = q.k / sqrt(hd), chunk max m,
//                    l = sum exp(s - m), acc = sum exp(s - m) v, all fp32 in
//                    ascending key order;
//   k_attn_merge:    per (row, query head): M = max m_c, L = sum exp(m_c - M) l_c,
//                    out = (sum exp(m_c - M) acc_c) / L * sigmoid(gate) -> bf16.
// The chunk width is a constant, so the partials of a row depend only on its
// own key count.
#pragma once

#include "common.cuh"

namespace hgd {

constexpr int ATTN_CHUNK = 32;  // keys per partial (one per lane)
constexpr int ATTN_MAX_HD = 256;
constexpr int ATTN_MAX_GROUP = 8;

struct AttnParams {
    const float* proj; int64_t proj_ld;  // rows: q (nq*hd) | gate (nq*hd) | k (nkv*hd) | v (nkv*hd)
    float* qrot;                         // [M][nq*hd]
    bf16_t* kcache; bf16_t* vcache;      // this layer: [B][nkv][Lmax][hd]
    const int32_t* pos;
    float* part;                         // [M][nq][max_chunks][hd + 2]
    bf16_t* out;                         // [M][nq*hd]
    int32_t* status;
    int B, T, nq, nkv, hd, Lmax, max_chunks;
    float rope_base;
};

// grid (M), block 256.
__global__ void __launch_bounds__(256) k_rope_append(const __grid_constant__ AttnParams p) {
    pdl_launch();
    pdl_wait();
    const int row = blockIdx.x;
    const int b = row / p.T, t = row % p.T;
    const int P = p.pos[b] + t;
    if (P < 0 || P >= p.Lmax) {
        if (threadIdx.x == 0) set_status(p.status, HGD_ERR_INVALID_ARG);
        return;
    }
    __shared__ float cs[ATTN_MAX_HD / 2], sn[ATTN_MAX_HD / 2];
    const int half = p.hd / 2;
    for (int i = threadIdx.x; i < half; i += blockDim.x) {
        // angle P * base^(-2i/hd) in double, reduced to [-pi, pi] in double, then
        // the fp32 sine and cosine of the reduced angle
        const double inv = exp2(-2.0 * (double)i / (double)p.hd * log2((double)p.rope_base));
        const double th = (double)P * inv;
        const double tw = 6.283185307179586476925286766559;
        const float r = (float)(th - tw * rint(th / tw));
        float s, c;
        sincosf(r, &s, &c);
        cs[i] = c;
        sn[i] = s;
    }
    __syncthreads();
    const float* pr = p.proj + (int64_t)row * p.proj_ld;
    const int qw = p.nq * p.hd;
    const float* kp = pr + 2 * qw;
    const float* vp = kp + p.nkv * p.hd;
    for (int e = threadIdx.x; e < (p.nq + p.nkv) * half; e += blockDim.x) {
        const int head = e / half, i = e % half;
        const float c = cs[i], s = sn[i];
        if (head < p.nq) {
            const float a = pr[head * p.hd + i], bb = pr[head * p.hd + i + half];
            float* qo = p.qrot + (int64_t)row * qw + head * p.hd;
            qo[i] = a * c - bb * s;
            qo[i + half] = bb * c + a * s;
        } else {
            const int g = head - p.nq;
            const float a = kp[g * p.hd + i], bb = kp[g * p.hd + i + half];
            bf16_t* ko = p.kcache + (((int64_t)b * p.nkv + g) * p.Lmax + P) * p.hd;
            ko[i] = f2bf(a * c - bb * s);
            ko[i + half] = f2bf(bb * c + a * s);
        }
    }
    for (int e = threadIdx.x; e < p.nkv * p.hd; e += blockDim.x) {
        const int g = e / p.hd, d = e % p.hd;
        p.vcache[(((int64_t)b * p.nkv + g) * p.Lmax + P) * p.hd + d] = f2bf(vp[e]);
    }
}

// grid (M, nkv, max_chunks), block 32 * group (one warp per query head of the
// group; group <= 8).  Chunk of ATTN_CHUNK (= 32) keys, one key per lane.
__global__ void __launch_bounds__(32 * ATTN_MAX_GROUP) k_attn_partial(const __grid_constant__ AttnParams p) {
    pdl_launch();
    pdl_wait();
    const int row = blockIdx.x, g = blockIdx.y, ch = blockIdx.z;
    const int b = row / p.T, t = row % p.T;
    const int P = p.pos[b] + t;
    if (P < 0 || P >= p.Lmax) return;
    const int key0 = ch * ATTN_CHUNK;
    if (key0 > P) return;
    const int nk = min(ATTN_CHUNK, P + 1 - key0);
    const int group = p.nq / p.nkv, hd = p.hd;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * group + warp;  // this warp's query head
    __shared__ float ex[ATTN_MAX_GROUP][ATTN_CHUNK];
    const bf16_t* K = p.kcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd;
    const bf16_t* V = p.vcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd;
    const float* q = p.qrot + (int64_t)row * p.nq * hd + (int64_t)h * hd;
    // scores: lane j takes key key0 + j; dot over hd in 8-element chunks, in order
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
    // chunk max and sum of exp (butterflies: order fixed by the lane pattern)
    float m = sc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float e = (lane < nk) ? expf(sc - m) : 0.f;
    const float l = warp_sum(e);
    ex[warp][lane] = e;
    __syncwarp();
    // acc[d] = sum_j e_j v_j[d]: lane owns dims 8*lane .. +7 (hd = 256) or a
    // strided set for smaller hd; keys in ascending order
    float* dst = p.part + (((int64_t)row * p.nq + h) * p.max_chunks + ch) * (hd + 2);
    for (int d0 = lane * 8; d0 < hd; d0 += 256) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < nk; ++j) {
            const uint4 vv = *reinterpret_cast<const uint4*>(V + (int64_t)(key0 + j) * hd + d0);
            const float w = ex[warp][j];
            acc[0] = fmaf(w, bf_lo(vv.x), acc[0]); acc[1] = fmaf(w, bf_hi(vv.x), acc[1]);
            acc[2] = fmaf(w, bf_lo(vv.y), acc[2]); acc[3] = fmaf(w, bf_hi(vv.y), acc[3]);
            acc[4] = fmaf(w, bf_lo(vv.z), acc[4]); acc[5] = fmaf(w, bf_hi(vv.z), acc[5]);
            acc[6] = fmaf(w, bf_lo(vv.w), acc[6]); acc[7] = fmaf(w, bf_hi(vv.w), acc[7]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[2 + d0 + i] = acc[i];
    }
    if (lane == 0) { dst[0] = m; dst[1] = l; }
}

// grid (M, nq), block hd.
__global__ void __launch_bounds__(256) k_attn_merge(const __grid_constant__ AttnParams p) {
    pdl_launch();
    pdl_wait();
    const int row = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
    const int b = row / p.T, t = row % p.T;
    const int P = p.pos[b] + t;
    const int hd = p.hd;
    bf16_t* out = p.out + (int64_t)row * p.nq * hd + (int64_t)h * hd;
    if (P < 0 || P >= p.Lmax) {
        if (d < hd) out[d] = 0;
        return;
    }
    const int nch = P / ATTN_CHUNK + 1;
    const float* base = p.part + ((int64_t)row * p.nq + h) * p.max_chunks * (hd + 2);
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, base[c * (hd + 2)]);
    float L = 0.f, acc = 0.f;
    for (int c = 0; c < nch; ++c) {
        const float* pc = base + c * (hd + 2);
        const float w = expf(pc[0] - M);
        L = fmaf(w, pc[1], L);
        if (d < hd) acc = fmaf(w, pc[2 + d], acc);
    }
    if (d < hd) {
        const float gate = p.proj[(int64_t)row * p.proj_ld + p.nq * hd + (int64_t)h * hd + d];
        out[d] = f2bf(acc / L * sigmoid_f(gate));
    }
}

}  // namespace hgd
