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

constexpr int ATTN_CHUNK = 64;
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
        const double th = (double)P * pow((double)p.rope_base, -2.0 * (double)i / (double)p.hd);
        double s, c;
        sincos(th, &s, &c);
        cs[i] = (float)c;
        sn[i] = (float)s;
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

// grid (M, nkv, max_chunks), block 128.
__global__ void __launch_bounds__(128) k_attn_partial(const __grid_constant__ AttnParams p) {
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
    __shared__ float qs[ATTN_MAX_GROUP][ATTN_MAX_HD];
    __shared__ float ex[ATTN_MAX_GROUP][ATTN_CHUNK];
    __shared__ float mls[ATTN_MAX_GROUP][2];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float* qrow = p.qrot + (int64_t)row * p.nq * hd + (int64_t)g * group * hd;
    for (int e = tid; e < group * hd; e += blockDim.x) qs[e / hd][e % hd] = qrow[e];
    __syncthreads();
    const float scale = 1.0f / sqrtf((float)hd);
    const bf16_t* K = p.kcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd;
    const bf16_t* V = p.vcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd;
    const int dpl = hd / 32;  // dims per lane (8 at hd = 256)
    for (int j = warp; j < nk; j += 4) {
        const bf16_t* kr = K + (int64_t)(key0 + j) * hd + lane * dpl;
        float kf[8];
        if (dpl == 8) {
            const uint4 v = *reinterpret_cast<const uint4*>(kr);
            kf[0] = bf_lo(v.x); kf[1] = bf_hi(v.x); kf[2] = bf_lo(v.y); kf[3] = bf_hi(v.y);
            kf[4] = bf_lo(v.z); kf[5] = bf_hi(v.z); kf[6] = bf_lo(v.w); kf[7] = bf_hi(v.w);
        } else {
            for (int e = 0; e < dpl; ++e) kf[e] = bf2f(kr[e]);
        }
        for (int hh = 0; hh < group; ++hh) {
            float d = 0.f;
            for (int e = 0; e < dpl; ++e) d = fmaf(qs[hh][lane * dpl + e], kf[e], d);
            d = warp_sum(d);
            if (lane == 0) ex[hh][j] = d * scale;
        }
    }
    __syncthreads();
    if (tid < group) {
        float m = -INFINITY;
        for (int j = 0; j < nk; ++j) m = fmaxf(m, ex[tid][j]);
        float l = 0.f;
        for (int j = 0; j < nk; ++j) {
            const float e = expf(ex[tid][j] - m);
            ex[tid][j] = e;
            l += e;
        }
        mls[tid][0] = m;
        mls[tid][1] = l;
    }
    __syncthreads();
    for (int hh = 0; hh < group; ++hh) {
        const int h = g * group + hh;
        float* dst = p.part + (((int64_t)row * p.nq + h) * p.max_chunks + ch) * (hd + 2);
        for (int d = tid; d < hd; d += blockDim.x) {
            float acc = 0.f;
            for (int j = 0; j < nk; ++j) acc = fmaf(ex[hh][j], bf2f(V[(int64_t)(key0 + j) * hd + d]), acc);
            dst[2 + d] = acc;
        }
        if (tid == 0) { dst[0] = mls[hh][0]; dst[1] = mls[hh][1]; }
    }
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
