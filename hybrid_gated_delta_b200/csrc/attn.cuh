// attn.cuh -- decode attention of the gated full-attention layers.
//
// "qwen3_5 cuda: mixed-width MLX checkpoints ... #849", PR body: gated attention
// with more query heads than key/value heads; partials over fixed-width key
// chunks plus a merge kernel with fp32 sums, the chunks cut at each key's
// logical position so that a row of a window sums exactly as its one-row step.
//
// Per row (stream b, window row t) at position P = pos[b] + t (the rotate-half
// RoPE of q and k at P and the append of K and V to the bf16 cache run in the
// in-projection's epilogue, gemv.cuh EPI_ROPE):
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
    const float* proj; int64_t proj_ld;  // rows: gate at columns nq*hd .. 2*nq*hd - 1
    const float* qrot;                   // [M][nq*hd] rotated queries
    bf16_t* kcache; bf16_t* vcache;      // this layer: [B][nkv][Lmax][hd]
    const int32_t* pos;
    float* part;                         // [M][nq][max_chunks][hd + 2]
    bf16_t* out;                         // [M][nq*hd]
    int32_t* status;
    int B, T, nq, nkv, hd, Lmax, max_chunks;
};

// One attention partial, computed by one warp: query q (fp32, rotated) over
// the nk keys key0 .. key0 + nk - 1 of one (stream, kv head) cache (K, V at
// position 0, rows of hd bf16).  Lane j scores key key0 + j (dot product over
// hd in ascending order, 8 elements at a time); chunk max m, l = sum exp(s - m),
// acc[d] = sum_j exp(s_j - m) v_j[d] in ascending key order.  dst: [hd + 2] =
// m, l, acc.  ex: 32 floats of this warp's shared scratch.
__device__ __forceinline__ void attn_partial_warp(const float* q, const bf16_t* K, const bf16_t* V, int key0,
                                                  int nk, int hd, float* dst, float* ex, int lane) {
    float sc = -INFINITY;
    if (lane < nk) {
        const bf16_t* kr = K + (int64_t)(key0 + lane) * hd;
        float d = 0.f;
#pragma unroll 8
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
    ex[lane] = e;
    __syncwarp();
    // acc[d]: lane owns dims 8*lane .. +7 (and +256 .. for larger hd); keys in order
    for (int d0 = lane * 8; d0 < hd; d0 += 256) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int j = 0; j < nk; ++j) {
            const uint4 vv = *reinterpret_cast<const uint4*>(V + (int64_t)(key0 + j) * hd + d0);
            const float w = ex[j];
            acc[0] = fmaf(w, bf_lo(vv.x), acc[0]); acc[1] = fmaf(w, bf_hi(vv.x), acc[1]);
            acc[2] = fmaf(w, bf_lo(vv.y), acc[2]); acc[3] = fmaf(w, bf_hi(vv.y), acc[3]);
            acc[4] = fmaf(w, bf_lo(vv.z), acc[4]); acc[5] = fmaf(w, bf_hi(vv.z), acc[5]);
            acc[6] = fmaf(w, bf_lo(vv.w), acc[6]); acc[7] = fmaf(w, bf_hi(vv.w), acc[7]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[2 + d0 + i] = acc[i];
    }
    if (lane == 0) { dst[0] = m; dst[1] = l; }
    __syncwarp();
}

// Merge of the nch chunk partials (rows of hd + 2 floats: m, l, acc) of one query
// head: M = max m_c; per dim d, L = sum exp(m_c - M) l_c and
// out = (sum exp(m_c - M) acc_c[d]) / L * sigmoid(gate), rounded to bf16.
__device__ __forceinline__ float attn_merge_max(const float* base, int nch, int hd) {
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, base[c * (hd + 2)]);
    return M;
}
__device__ __forceinline__ bf16_t attn_merge_dim(const float* base, int nch, int hd, float M, int d, float gate) {
    float L = 0.f, acc = 0.f;
#pragma unroll 4
    for (int c = 0; c < nch; ++c) {
        const float* pc = base + c * (hd + 2);
        const float w = expf(pc[0] - M);
        L = fmaf(w, pc[1], L);
        acc = fmaf(w, pc[2 + d], acc);
    }
    return f2bf(acc / L * sigmoid_f(gate));
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
    float* dst = p.part + (((int64_t)row * p.nq + h) * p.max_chunks + ch) * (hd + 2);
    attn_partial_warp(q, K, V, key0, nk, hd, dst, ex[warp], lane);
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
    if (d >= hd) return;
    const int nch = P / ATTN_CHUNK + 1;
    const float* base = p.part + ((int64_t)row * p.nq + h) * p.max_chunks * (hd + 2);
    const float M = attn_merge_max(base, nch, hd);
    const float gate = p.proj[(int64_t)row * p.proj_ld + p.nq * hd + (int64_t)h * hd + d];
    out[d] = attn_merge_dim(base, nch, hd, M, d, gate);
}

}  // namespace hgd
