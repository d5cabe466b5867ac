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
//                    heads of the group: s = q.k / sqrt(hd) (each lane's share
//                    of the dims, then a butterfly over the lanes), chunk max
//                    m, l = sum exp(s - m), acc = sum exp(s - m) v, fp32, the
//                    sums over keys in ascending key order;
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
    int pack_ntp;  // > 0: out holds the rows packed for the tensor-core GEMM (tc_x_elem, NTp rows)
};

// One attention partial, computed by one warp: query q (fp32, rotated) over
// the nk <= 32 keys key0 .. key0 + nk - 1 of one (stream, kv head) cache (K, V
// at position 0, rows of hd bf16).  Lane l owns the DPL = hd / 32 contiguous
// dims [l*DPL, (l+1)*DPL): per key it forms its share of q.k (fmaf over its
// dims in order) and a butterfly over the lanes completes the dot product;
// s_j = dot / sqrt(hd), chunk max m, l = sum_j exp(s_j - m) (butterfly),
// acc[d] = sum_j exp(s_j - m) v_j[d] in ascending key order.  Key and value
// rows load coalesced, 16 keys at a time.  dst: [hd + 2] = m, l, acc.
// DPL consecutive bf16 of a cache row, packed two per word (DPL = 1: one).
template <int DPL>
struct AttnRow { uint32_t w[(DPL + 1) / 2]; };
template <int DPL>
__device__ __forceinline__ AttnRow<DPL> attn_rowload(const bf16_t* row) {
    AttnRow<DPL> r;
    if (DPL == 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(row);
        r.w[0] = u.x; r.w[1] = u.y; r.w[2] = u.z; r.w[3] = u.w;
    } else if (DPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(row);
        r.w[0] = u.x; r.w[1] = u.y;
    } else if (DPL == 2) {
        r.w[0] = *reinterpret_cast<const uint32_t*>(row);
    } else {
        r.w[0] = (uint32_t)row[0];
    }
    return r;
}
template <int DPL>
__device__ __forceinline__ float attn_elem(const AttnRow<DPL>& r, int i) {
    return (i & 1) ? bf_hi(r.w[i >> 1]) : bf_lo(r.w[i >> 1]);
}

// PF: K and V are in global memory and this lane's share of the chunk is
// prefetched into L1 first; without it they may be shared-memory rows.
template <int DPL, bool PF = true>
__device__ void attn_partial_warp_t(const float* q, const bf16_t* K, const bf16_t* V, int key0, int nk, float* dst,
                                    int lane) {
    constexpr int hd = 32 * DPL, KB = 16;
    const int d0 = lane * DPL;
    // this lane's share of every key and value row of the chunk into L1 now, so
    // the loads below (keys in two batches, then values after the softmax) hit it
    if (PF)
        for (int j = 0; j < nk; ++j) {
            prefetch_l1(K + (int64_t)(key0 + j) * hd + d0);
            prefetch_l1(V + (int64_t)(key0 + j) * hd + d0);
        }
    float qv[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) qv[i] = q[d0 + i];
    // this lane's share of every key's dot product, then all 32 summed over the
    // lanes at once (warp_sum_transposed: warp_sum's pairings, so each score is
    // bitwise warp_sum's), which leaves key j's in lane j
    float dd[32];
#pragma unroll
    for (int b = 0; b < 32; b += KB) {
        AttnRow<DPL> kr[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            if (b + j < nk) kr[j] = attn_rowload<DPL>(K + (int64_t)(key0 + b + j) * hd + d0);
            else {
#pragma unroll
                for (int i = 0; i < (DPL + 1) / 2; ++i) kr[j].w[i] = 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            dd[b + j] = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) dd[b + j] = fmaf(qv[i], attn_elem<DPL>(kr[j], i), dd[b + j]);
        }
    }
    const float tot = warp_sum_transposed<32>(dd, lane);
    const float sc = lane < nk ? tot * (1.0f / sqrtf((float)hd)) : -INFINITY;  // lane j: key j's scaled score
    float m = sc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float e = (lane < nk) ? expf(sc - m) : 0.f;
    const float l = warp_sum(e);
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll
    for (int b = 0; b < 32; b += KB) {
        if (b >= nk) break;
        AttnRow<DPL> vr[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            if (b + j < nk) vr[j] = attn_rowload<DPL>(V + (int64_t)(key0 + b + j) * hd + d0);
            else {
#pragma unroll
                for (int i = 0; i < (DPL + 1) / 2; ++i) vr[j].w[i] = 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const float w = __shfl_sync(0xffffffffu, e, b + j);
            if (b + j < nk) {
#pragma unroll
                for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, attn_elem<DPL>(vr[j], i), acc[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[2 + d0 + i] = acc[i];
    if (lane == 0) { dst[0] = m; dst[1] = l; }
    __syncwarp();
}

// Two query heads of one row over one chunk whose key and value rows sit in
// shared memory (K, V at the chunk's first key), by one warp: every key and
// value row is read and unpacked once for both heads.  Per head the arithmetic
// of attn_partial_warp_t: the same fmaf order per key, and every sum over the
// lanes with warp_sum's pairings (the scores summed 16 keys at a time by
// warp_sum_transposed, then moved to lane j), so each partial is bitwise its.
template <int DPL>
__device__ void attn_partial_pair(const float* q0, const float* q1, const bf16_t* K, const bf16_t* V, int nk,
                                  float* dst0, float* dst1, int lane) {
    constexpr int hd = 32 * DPL, KB = 16;
    const int d0 = lane * DPL;
    float qa[DPL], qb[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) { qa[i] = q0[d0 + i]; qb[i] = q1[d0 + i]; }
    float ta[2], tb[2];  // batch bi: key (lane >> 1) of the batch, summed over the lanes
#pragma unroll
    for (int bi = 0; bi < 2; ++bi) {
        const int b = bi * KB;
        AttnRow<DPL> kr[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            if (b + j < nk) kr[j] = attn_rowload<DPL>(K + (int64_t)(b + j) * hd + d0);
            else {
#pragma unroll
                for (int i = 0; i < (DPL + 1) / 2; ++i) kr[j].w[i] = 0u;
            }
        }
        float da[KB], db[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            da[j] = 0.f;
            db[j] = 0.f;
#pragma unroll
            for (int i = 0; i < DPL; ++i) {
                const float kv = attn_elem<DPL>(kr[j], i);
                da[j] = fmaf(qa[i], kv, da[j]);
                db[j] = fmaf(qb[i], kv, db[j]);
            }
        }
        ta[bi] = warp_sum_transposed<KB>(da, lane);
        tb[bi] = warp_sum_transposed<KB>(db, lane);
    }
    // key L's sum to lane L: batch L >> 4 holds it in lanes 2 (L & 15), 2 (L & 15) + 1
    const int src = 2 * (lane & 15);
    const float xa0 = __shfl_sync(0xffffffffu, ta[0], src), xa1 = __shfl_sync(0xffffffffu, ta[1], src);
    const float xb0 = __shfl_sync(0xffffffffu, tb[0], src), xb1 = __shfl_sync(0xffffffffu, tb[1], src);
    const float sa = lane < nk ? (lane < KB ? xa0 : xa1) * (1.0f / sqrtf((float)hd)) : -INFINITY;
    const float sb = lane < nk ? (lane < KB ? xb0 : xb1) * (1.0f / sqrtf((float)hd)) : -INFINITY;
    float ma = sa, mb = sb;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
    }
    const float ea = (lane < nk) ? expf(sa - ma) : 0.f, eb = (lane < nk) ? expf(sb - mb) : 0.f;
    const float la = warp_sum(ea), lb = warp_sum(eb);
    float acca[DPL], accb[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) { acca[i] = 0.f; accb[i] = 0.f; }
#pragma unroll
    for (int b = 0; b < 32; b += KB) {
        if (b >= nk) break;
        AttnRow<DPL> vr[KB];
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            if (b + j < nk) vr[j] = attn_rowload<DPL>(V + (int64_t)(b + j) * hd + d0);
            else {
#pragma unroll
                for (int i = 0; i < (DPL + 1) / 2; ++i) vr[j].w[i] = 0u;
            }
        }
#pragma unroll
        for (int j = 0; j < KB; ++j) {
            const float wa = __shfl_sync(0xffffffffu, ea, b + j), wb = __shfl_sync(0xffffffffu, eb, b + j);
            if (b + j < nk) {
#pragma unroll
                for (int i = 0; i < DPL; ++i) {
                    const float vv = attn_elem<DPL>(vr[j], i);
                    acca[i] = fmaf(wa, vv, acca[i]);
                    accb[i] = fmaf(wb, vv, accb[i]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) { dst0[2 + d0 + i] = acca[i]; dst1[2 + d0 + i] = accb[i]; }
    if (lane == 0) { dst0[0] = ma; dst0[1] = la; dst1[0] = mb; dst1[1] = lb; }
    __syncwarp();
}

// hd = 32 * DPL with DPL one of 1, 2, 4, 8 (the shapes check_supported admits).
__device__ __forceinline__ void attn_partial_warp(const float* q, const bf16_t* K, const bf16_t* V, int key0,
                                                  int nk, int hd, float* dst, int lane) {
    switch (hd) {
        case 256: attn_partial_warp_t<8>(q, K, V, key0, nk, dst, lane); break;
        case 128: attn_partial_warp_t<4>(q, K, V, key0, nk, dst, lane); break;
        case 64: attn_partial_warp_t<2>(q, K, V, key0, nk, dst, lane); break;
        default: attn_partial_warp_t<1>(q, K, V, key0, nk, dst, lane); break;
    }
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

// grid (B, nkv, max_chunks), block 256: one CTA per (stream, kv head, chunk of
// ATTN_CHUNK keys) stages the chunk's key and value rows in shared memory once,
// then its eight warps take the (row, query head) pairs of the stream's T rows
// whose position reaches the chunk, each with attn_partial_warp_t's arithmetic
// (the same partial, bit for bit, as one warp per pair reading the cache).
constexpr int ATTN_PART_WARPS = 8;
__host__ __device__ inline size_t attn_part_smem_bytes(int hd) { return (size_t)2 * ATTN_CHUNK * hd * 2; }
__global__ void __launch_bounds__(32 * ATTN_PART_WARPS) k_attn_partial(const __grid_constant__ AttnParams p) {
    extern __shared__ __align__(16) uint8_t attn_smem[];
    pdl_launch();
    pdl_wait();
    const int b = blockIdx.x, g = blockIdx.y, ch = blockIdx.z, hd = p.hd;
    const int key0 = ch * ATTN_CHUNK, pos = p.pos[b];
    // the rows of this stream with a valid position that reaches the chunk
    int tlo = max(0, key0 - pos), thi = min(p.T, p.Lmax - pos);
    if (pos < 0) tlo = max(tlo, -pos);
    if (tlo >= thi) return;
    const int nkc = min(ATTN_CHUNK, pos + thi - key0);  // keys the chunk's last row sees
    const bf16_t* K = p.kcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd + (int64_t)key0 * hd;
    const bf16_t* V = p.vcache + ((int64_t)b * p.nkv + g) * p.Lmax * hd + (int64_t)key0 * hd;
    bf16_t* Ks = reinterpret_cast<bf16_t*>(attn_smem);
    bf16_t* Vs = Ks + ATTN_CHUNK * hd;
    const int n16 = nkc * hd / 8;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) {
        reinterpret_cast<uint4*>(Ks)[i] = reinterpret_cast<const uint4*>(K)[i];
        reinterpret_cast<uint4*>(Vs)[i] = reinterpret_cast<const uint4*>(V)[i];
    }
    __syncthreads();
    const int group = p.nq / p.nkv, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if ((group & 1) == 0) {  // head pairs: the chunk's rows read once for two heads
        const int hp = group / 2;
        for (int pi = tlo * hp + warp; pi < thi * hp; pi += ATTN_PART_WARPS) {
            const int t = pi / hp, h = g * group + 2 * (pi % hp), row = b * p.T + t;
            const int nk = min(ATTN_CHUNK, pos + t + 1 - key0);
            const float* q = p.qrot + (int64_t)row * p.nq * hd + (int64_t)h * hd;
            float* dst = p.part + (((int64_t)row * p.nq + h) * p.max_chunks + ch) * (hd + 2);
            float* dst1 = dst + (int64_t)p.max_chunks * (hd + 2);  // head h + 1
            switch (hd) {
                case 256: attn_partial_pair<8>(q, q + hd, Ks, Vs, nk, dst, dst1, lane); break;
                case 128: attn_partial_pair<4>(q, q + hd, Ks, Vs, nk, dst, dst1, lane); break;
                case 64: attn_partial_pair<2>(q, q + hd, Ks, Vs, nk, dst, dst1, lane); break;
                default: attn_partial_pair<1>(q, q + hd, Ks, Vs, nk, dst, dst1, lane); break;
            }
        }
        return;
    }
    for (int pi = tlo * group + warp; pi < thi * group; pi += ATTN_PART_WARPS) {
        const int t = pi / group, h = g * group + pi % group, row = b * p.T + t;
        const int nk = min(ATTN_CHUNK, pos + t + 1 - key0);
        const float* q = p.qrot + (int64_t)row * p.nq * hd + (int64_t)h * hd;
        float* dst = p.part + (((int64_t)row * p.nq + h) * p.max_chunks + ch) * (hd + 2);
        switch (hd) {
            case 256: attn_partial_warp_t<8, false>(q, Ks, Vs, 0, nk, dst, lane); break;
            case 128: attn_partial_warp_t<4, false>(q, Ks, Vs, 0, nk, dst, lane); break;
            case 64: attn_partial_warp_t<2, false>(q, Ks, Vs, 0, nk, dst, lane); break;
            default: attn_partial_warp_t<1, false>(q, Ks, Vs, 0, nk, dst, lane); break;
        }
    }
}

// grid (M, nq), block hd: the merge of attn_merge_max / attn_merge_dim, with
// every load issued up front (thread c: chunk c's m and l; thread d: its gate
// and the first ATTN_MERGE_Q chunks' values of dim d) and w_c = exp(m_c - M)
// formed once per chunk into shared memory; max is exact and w_c the same
// expression, so the result is theirs bit for bit.
constexpr int ATTN_MERGE_Q = 24;
constexpr int ATTN_MAX_CHUNKS = 512;  // positions up to 16384
__global__ void __launch_bounds__(256) k_attn_merge(const __grid_constant__ AttnParams p) {
    __shared__ float wv[ATTN_MAX_CHUNKS], lv[ATTN_MAX_CHUNKS], wm[8];
    pdl_launch();
    pdl_wait();
    const int row = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
    const int b = row / p.T, t = row % p.T;
    const int P = p.pos[b] + t;
    const int hd = p.hd;
    bf16_t* out = p.pack_ntp ? p.out + tc_x_elem(row, h * hd + d, p.pack_ntp)
                             : p.out + (int64_t)row * p.nq * hd + (int64_t)h * hd + d;
    if (P < 0 || P >= p.Lmax) {
        if (d < hd) *out = 0;
        return;
    }
    const int nch = P / ATTN_CHUNK + 1;
    const float* base = p.part + ((int64_t)row * p.nq + h) * p.max_chunks * (hd + 2);
    float a[ATTN_MERGE_Q];
    float gate = 0.f;
    if (d < hd) {
        gate = p.proj[(int64_t)row * p.proj_ld + p.nq * hd + (int64_t)h * hd + d];
#pragma unroll
        for (int c = 0; c < ATTN_MERGE_Q; ++c) a[c] = c < nch ? base[c * (hd + 2) + 2 + d] : 0.f;
    }
    float mx = -INFINITY;
    for (int c = d; c < nch; c += blockDim.x) {
        const float2 ml = *reinterpret_cast<const float2*>(base + c * (hd + 2));
        wv[c] = ml.x;
        lv[c] = ml.y;
        mx = fmaxf(mx, ml.x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((d & 31) == 0) wm[d >> 5] = mx;
    __syncthreads();
    float M = wm[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) M = fmaxf(M, wm[w]);
    for (int c = d; c < nch; c += blockDim.x) wv[c] = expf(wv[c] - M);
    __syncthreads();
    if (d >= hd) return;
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int c = 0; c < ATTN_MERGE_Q; ++c)
        if (c < nch) {
            L = fmaf(wv[c], lv[c], L);
            acc = fmaf(wv[c], a[c], acc);
        }
    for (int c0 = ATTN_MERGE_Q; c0 < nch; c0 += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = c0 + u < nch ? base[(c0 + u) * (hd + 2) + 2 + d] : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
            if (c0 + u < nch) {
                L = fmaf(wv[c0 + u], lv[c0 + u], L);
                acc = fmaf(wv[c0 + u], v[u], acc);
            }
    }
    *out = f2bf(acc / L * sigmoid_f(gate));
}

}  // namespace hgd
