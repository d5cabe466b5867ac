// Tensor-core GEMM for windows of token rows (tcgen05, sm_100a):
//
//   Y[t][n] = sum_k X[t][k] * W[n][k]     t < M <= 256 token rows, fp32 sums
//
// The decode-step projections of the hybrid stack (Qwen3.5-style gated-delta /
// gated-attention decoder; the projection GEMVs of the decode step) become real
// GEMMs once a call carries a window of many token rows: at 128 rows a weight
// byte feeds 128 multiply-adds, which the legacy mma.sync path cannot sustain.
// Here one CTA owns a 128-row block of W (the MMA's M), takes every token row
// of the call as the MMA's N (16..256), and streams its K range through a ring
// of shared-memory stages:
//   - one lane issues the bulk copies (cp.async.bulk, into this CTA only) of a
//     stage's weight tile (128 x 64, 16 KB) and token tile (NTp x 64),
//     completing on the stage's `full` mbarrier;
//   - one lane issues four tcgen05.mma (K = 16 each) per stage into a TMEM
//     accumulator of 128 lanes x NTp fp32 columns, and tcgen05.commit frees the
//     stage (`empty`) once they complete;
//   - after the last stage, the four warps read the accumulator back with
//     tcgen05.ld (warp w owns TMEM lanes 32w..32w+31 = W rows) and write fp32.
// Operands are packed once into the canonical no-swizzle K-major layout the
// shared-memory descriptors describe: 8 x 8 core matrices (8 rows of 16 bytes,
// 128 contiguous bytes), core (row group g, k group j) of a tile at byte
// (g * 8 + j) * 128, so the leading-dimension (k) stride is 128 bytes and the
// stride-dimension (8-row group) stride is 1024 bytes.  A fixed split of K over
// CTAs (a function of N and K only, at most 8) fills the SMs for short-N
// projections.  The splits of a 128-row block run as one thread-block cluster:
// each CTA parks its accumulator in its own shared memory, and after a cluster
// barrier CTA r sums the r-th share of the token rows over the cluster's
// shared memories in split order and writes it, so the partials never leave
// the SMs.  The epilogue writes fp32 rows or adds them to bf16 residual rows.
//
// Every wait is bounded (HGD_ERR_TIMEOUT in *status), the producer waits for
// its copies before the CTA leaves, the issuer's final commit covers every MMA
// it issued, and the TMEM columns are freed on every path.
#pragma once
#include "common.cuh"

namespace hgd {

constexpr int TC_BM = 128;                    // W rows per tile (the MMA's M)
constexpr int TC_MAXN = 256;                  // token rows per call (the MMA's N)
constexpr int TC_THREADS = 256;  // warp 0 lane 0: copies, warp 1 lane 0: MMAs; all eight: the epilogue
constexpr int TC_WTILE = TC_BM * TC_BK;       // elements of a weight tile (16 KB)
constexpr int TC_MAX_STAGES = 8;
constexpr int TC_TARGET_CTAS = 148;           // split-K target: one wave of B200 SMs
constexpr int TC_MAX_SPLITS = 8;              // a portable cluster

__host__ __device__ inline int tc_ntp(int M) { return M <= 16 ? 16 : (M + 15) / 16 * 16; }
__host__ __device__ inline int tc_nblocks(int N) { return (N + TC_BM - 1) / TC_BM; }

// Packed weight: tile (n / 128, k / 64) at tile index nb * (K / 64) + kb, each
// tile in core-matrix order.  Element offset of W[n][k]:
__host__ __device__ inline size_t tc_w_elem(int n, int k, int K) {
    const int r = n & (TC_BM - 1), kk = k & (TC_BK - 1);
    const size_t tile = (size_t)(n >> 7) * (K / TC_BK) + (k >> 6);
    return tile * TC_WTILE + (size_t)(((r >> 3) * 8 + (kk >> 3)) * 64 + (r & 7) * 8 + (kk & 7));
}
// Packed token rows: tc_x_elem (common.cuh), the same core order per k block.

// One 16-byte chunk (8 consecutive k) per thread: rows n >= N are zero.
__global__ void k_tc_pack_w(const bf16_t* __restrict__ W, bf16_t* __restrict__ Wp, int N, int K) {
    const int cpr = K / 8;
    const int64_t total = (int64_t)tc_nblocks(N) * TC_BM * cpr;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(e / cpr), k = (int)(e % cpr) * 8;
        const uint4 v = n < N ? *reinterpret_cast<const uint4*>(W + (int64_t)n * K + k) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(Wp + tc_w_elem(n, k, K)) = v;
    }
}
// The gate (half 0) or up (half 1) rows [N, K] of a SwiGLU projection into the
// interleaved packed matrix: source row n goes to row (n / 64) * 128 + half * 64
// + n % 64; rows past N are zero.
__global__ void k_tc_pack_w_swiglu(const bf16_t* __restrict__ W, bf16_t* __restrict__ Wp, int N, int K, int half) {
    const int cpr = K / 8;
    const int64_t total = (int64_t)((N + 63) / 64) * 64 * cpr;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(e / cpr), k = (int)(e % cpr) * 8;
        const uint4 v = n < N ? *reinterpret_cast<const uint4*>(W + (int64_t)n * K + k) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(Wp + tc_w_elem((n >> 6) * 128 + half * 64 + (n & 63), k, K)) = v;
    }
}
__global__ void k_tc_pack_x(const bf16_t* __restrict__ X, int64_t x_ld, bf16_t* __restrict__ Xp, int M, int K,
                            int NTp) {
    pdl_launch();
    pdl_wait();
    const int cpr = K / 8;
    const int total = NTp * cpr;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
        const int t = e / cpr, k = (e % cpr) * 8;
        const uint4 v = t < M ? *reinterpret_cast<const uint4*>(X + (int64_t)t * x_ld + k) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(Xp + tc_x_elem(t, k, NTp)) = v;
    }
}

// ------------------------------------------------------------- tcgen05 PTX
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Shared-memory matrix descriptor: no swizzle, K-major, start / leading (k) /
// stride (8-row group) byte offsets in 16-byte units, descriptor version 1.
__device__ __forceinline__ uint64_t tc_desc(const void* smem, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((smem_addr(smem) >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::f16: bf16 A and B, both K-major, fp32 D,
// M = 128, N = n.
__host__ __device__ inline uint32_t tc_idesc(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every MMA this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct TcParams {
    const bf16_t* Wp;   // packed weight (tc_w_elem), N padded to 128-row tiles
    const bf16_t* Xp;   // packed token rows (tc_x_elem), NTp rows
    float* out;         // Y [M][ldo] (fp32), when resid and h are null
    bf16_t* resid;      // or: resid[t][n] = bf16(resid[t][n] + Y[t][n]), [M][ldo]
    bf16_t* h;          // or (SwiGLU): W holds gate and up rows interleaved by 64 (k_tc_pack_w_swiglu);
    int I;              //   h[t][i] = bf16(silu(gate_i) * up_i), i < I, packed (tc_x_elem, NTp rows)
    int32_t* status;    // optional: HGD_ERR_TIMEOUT if a wait ran out
    int M, N, K, NTp, ldo;
    int n_blocks, kb_per_split, splits, stages;  // splits: the cluster size (1: no cluster)
    int wpb;            // 128-row weight blocks per CTA (2: two accumulators share each token tile; splits 1)
    int npair;          // wpb 2: CTAs [0, npair) own block pairs, the later CTAs one block each
    uint32_t tmem_cols;
};

// ------------------------------------------------ cluster shared memory
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
// Bulk copy (the async proxy) of `bytes` from this CTA's shared memory to shared
// memory of a CTA of the cluster, completing `bytes` of transaction count on that
// CTA's mbarrier (dst and mbar: cluster addresses, dsmem_addr).  No multicast.
__device__ __forceinline__ void bulk_s2cluster(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(smem_addr(src)), "r"(bytes), "r"(mbar)
                 : "memory");
}
// Generic-proxy writes to shared memory made visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ int ld_dsmem_s32(uint32_t a) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
// SwiGLU of token rows t_lo.. t_hi - 1 of row block nb from st (row t at
// st[(t - t_lo) * 128 ..]: 64 gate rows, then the 64 matching up rows).
__device__ __forceinline__ void tc_swiglu_rows(const TcParams& p, const float* st, int t_lo, int t_hi, int nb,
                                               int tid) {
#pragma unroll 4
    for (int e = tid; e < (t_hi - t_lo) * 64; e += TC_THREADS) {
        const int tt = e >> 6, il = e & 63, i = nb * 64 + il, t = t_lo + tt;
        if (i < p.I && t < p.M)
            p.h[tc_x_elem(t, i, p.NTp)] = f2bf(silu_f(st[tt * TC_BM + il]) * st[tt * TC_BM + 64 + il]);
    }
}
// The split sum of this CTA's token rows t_lo .. t_hi - 1 of one pass: red holds
// split sp's own partials ([t][row]), rcv the others' (slot per sender), summed
// in split order, four rows per thread (float4), eight token lanes.  The sums go
// back into red (SwiGLU), onto the bf16 residual, or out as fp32.
template <int SPLITS>
__device__ __forceinline__ void tc_split_sum(const TcParams& p, float* red, const float* rcv, int per, int sp,
                                             int t_lo, int t_hi, int tq, int nb, int tid, bool vec) {
    const int q4 = tid & 31, tl = tid >> 5, nn = nb * TC_BM + 4 * q4;
#pragma unroll 2
    for (int t = t_lo + tl; t < t_hi; t += TC_THREADS / 32) {
        float4 v[SPLITS];
#pragma unroll
        for (int r = 0; r < SPLITS; ++r) {
            const float* src = r == sp ? red + (size_t)t * TC_BM
                                       : rcv + ((size_t)(r < sp ? r : r - 1) * per + (t - t_lo)) * TC_BM;
            v[r] = *reinterpret_cast<const float4*>(src + 4 * q4);
        }
        float4 a = v[0];
#pragma unroll
        for (int r = 1; r < SPLITS; ++r) { a.x += v[r].x; a.y += v[r].y; a.z += v[r].z; a.w += v[r].w; }
        if (p.h) {
            *reinterpret_cast<float4*>(red + (size_t)t * TC_BM + 4 * q4) = a;  // this CTA's own rows
            continue;
        }
        const size_t e = (size_t)(tq + t) * p.ldo + nn;
        const float av[4] = {a.x, a.y, a.z, a.w};
        if (vec && nn + 3 < p.N) {
            if (p.resid) {
                const uint2 r2 = *reinterpret_cast<const uint2*>(p.resid + e);
                *reinterpret_cast<uint2*>(p.resid + e) =
                    make_uint2(pack_bf2(bf_lo(r2.x) + av[0], bf_hi(r2.x) + av[1]),
                               pack_bf2(bf_lo(r2.y) + av[2], bf_hi(r2.y) + av[3]));
            } else {
                *reinterpret_cast<float4*>(p.out + e) = a;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (nn + j < p.N) {
                    if (p.resid) p.resid[e + j] = f2bf(bf2f(p.resid[e + j]) + av[j]);
                    else p.out[e + j] = av[j];
                }
        }
    }
}
__device__ __forceinline__ void tc_store(const TcParams& p, int t, int n, float v) {
    const size_t e = (size_t)t * p.ldo + n;
    if (p.resid) p.resid[e] = f2bf(bf2f(p.resid[e]) + v);
    else p.out[e] = v;
}

// Shared memory: stages x (weight tile 16 KB, token tile NTp x 128 B), then the
// full / empty / done mbarriers, the TMEM address and the abort flag.  With
// splits, the stages then hold the accumulator (NTp x 128 fp32, tc_red_bytes):
// the plan gives enough stages for it.
__host__ __device__ inline size_t tc_stage_bytes(int NTp, int wpb = 1) {
    return (size_t)wpb * TC_WTILE * 2 + (size_t)NTp * TC_BK * 2;
}
// The split epilogue works on up to TC_RED_T token rows at a time.  Shared
// memory it needs in the stages: the pass's accumulator rows, then the other
// splits' partials of this CTA's share of them.
constexpr int TC_RED_T = 128;
__host__ __device__ inline size_t tc_red_bytes(int NTp, int splits) {
    const int rows = NTp < TC_RED_T ? NTp : TC_RED_T;
    return (size_t)rows * TC_BM * 4 + (size_t)(splits - 1) * (rows / splits) * TC_BM * 4;
}
__host__ __device__ inline size_t tc_smem_bytes(int NTp, int stages, int wpb = 1) {
    return (size_t)stages * tc_stage_bytes(NTp, wpb) + (2 * TC_MAX_STAGES + 1) * 8 + 32;
}

__global__ void __launch_bounds__(TC_THREADS, 1) k_gemm_tc(const __grid_constant__ TcParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.stages;
    const size_t sb = tc_stage_bytes(p.NTp, p.wpb);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * sb);
    uint64_t* empty = full + TC_MAX_STAGES;
    uint64_t* done = empty + TC_MAX_STAGES;
    volatile uint32_t* tslot = reinterpret_cast<volatile uint32_t*>(done + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(done + 1) + 1;
    uint64_t* rbar = done + 3;  // the split epilogue: the other splits' partials have landed
    // the splits of a row block are consecutive CTAs, one cluster: sp is the rank;
    // with wpb = 2 the first npair CTAs own blocks nb and nb + 1 and the rest one
    // block each, so the last wave of CTAs is made of short ones
    const int cta = blockIdx.x / p.splits, sp = blockIdx.x % p.splits;
    const int nb = p.wpb == 2 ? (cta < p.npair ? 2 * cta : 2 * p.npair + (cta - p.npair)) : cta;
    const int wn = p.wpb == 2 ? min(cta < p.npair ? 2 : 1, p.n_blocks - nb) : 1;  // weight blocks of this CTA
    const int nkb_all = p.K / TC_BK;
    const int kb0 = sp * p.kb_per_split, nkb = max(0, min(nkb_all, kb0 + p.kb_per_split) - kb0);

    const uint32_t xbytes = (uint32_t)p.NTp * TC_BK * 2, wbytes = (uint32_t)TC_WTILE * 2;
    const int pre = min(S, nkb);
    if (tid == 0) {
        for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        mbar_init(done, 1);
        mbar_init(rbar, 1);
        *abort_flag = 0;
        mbar_fence_init();
        // the first stages' weight tiles go out at once, by the thread that set up
        // their barriers, before the TMEM allocation and the CTA barrier (weights
        // are never written by the previous kernel on the stream); their token
        // tiles follow the wait for that kernel
        const uint64_t pol_w = policy_evict_first();
        for (int i = 0; i < pre; ++i) {
            mbar_arrive_expect_tx(&full[i], (uint32_t)wn * wbytes + xbytes);
            for (int j = 0; j < wn; ++j)
                bulk_g2s(smem + (size_t)i * sb + j * wbytes, p.Wp + ((size_t)(nb + j) * nkb_all + kb0 + i) * TC_WTILE,
                         wbytes, &full[i], pol_w);
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(const_cast<uint32_t*>(tslot))),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    pdl_launch();

    if (warp == 0 && lane == 0) {
        // producer (the same thread): the first stages' token tiles after the wait
        // for the previous kernel; then stage by stage as the MMAs free them
        const uint32_t xoff = (uint32_t)p.wpb * wbytes;  // the token tile follows the weight tiles
        const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
        pdl_wait();
        for (int i = 0; i < pre; ++i)
            bulk_g2s(smem + (size_t)i * sb + xoff, p.Xp + (size_t)(kb0 + i) * p.NTp * TC_BK, xbytes, &full[i],
                     pol_x);
        int issued = pre;
        bool ok = true;
        for (int i = pre; i < nkb; ++i) {
            const int st = i % S;
            if (!mbar_wait_bounded(&empty[st], (uint32_t)(((i / S) & 1) ^ 1), abort_flag)) {
                ok = false;
                break;
            }
            mbar_arrive_expect_tx(&full[st], (uint32_t)wn * wbytes + xbytes);
            uint8_t* dst = smem + (size_t)st * sb;
            for (int j = 0; j < wn; ++j)
                bulk_g2s(dst + j * wbytes, p.Wp + ((size_t)(nb + j) * nkb_all + kb0 + i) * TC_WTILE, wbytes, &full[st],
                         pol_w);
            bulk_g2s(dst + xoff, p.Xp + (size_t)(kb0 + i) * p.NTp * TC_BK, xbytes, &full[st], pol_x);
            issued = i + 1;
        }
        if (!ok) {
            if (p.status) set_status(p.status, HGD_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        // the copies still in flight land before this CTA's shared memory goes away
        for (int q = max(0, issued - S); q < issued; ++q)
            (void)mbar_wait_bounded(&full[q % S], (uint32_t)((q / S) & 1), nullptr);
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        const uint32_t idesc = tc_idesc(p.NTp);
        for (int i = 0; i < nkb; ++i) {
            const int st = i % S;
            if (!mbar_wait_bounded(&full[st], (uint32_t)((i / S) & 1), abort_flag)) {
                if (p.status) set_status(p.status, HGD_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint8_t* a = smem + (size_t)st * sb;
            const uint8_t* b = a + (size_t)p.wpb * TC_WTILE * 2;
            // weight block j accumulates in TMEM columns j * 128 .. (NTp <= 128 with wpb = 2)
            for (int j = 0; j < wn; ++j)
#pragma unroll
                for (int s = 0; s < TC_BK / 16; ++s)
                    tc_mma(tmem + (uint32_t)(j * 128), tc_desc(a + (size_t)j * TC_WTILE * 2 + s * 256, 128, 1024),
                           tc_desc(b + s * 256, 128, 1024), idesc, (i > 0 || s > 0) ? 1u : 0u);
            tc_commit(&empty[st]);
        }
        tc_commit(done);  // covers every MMA issued above
    }
    __syncwarp();

    // epilogue: warp w reads TMEM lanes 32w.. (W rows nb*128 + 32w + lane)
    const bool got = mbar_wait_bounded(done, 0u, nullptr);
    tc_fence_after();
    if (!got && lane == 0 && p.status) set_status(p.status, HGD_ERR_TIMEOUT);
    const bool good = __syncthreads_and(got && !*abort_flag);  // no wait of this CTA ran out
    const bool live = good && nkb > 0;
    // warp w reads TMEM lane quarter w & 3 (W rows 32 (w & 3) + lane of a block) and
    // half w >> 2 of the accumulator's columns (token rows)
    const int lq = warp & 3, ch = warp >> 2;
    const int n = nb * TC_BM + lq * 32 + lane;
    auto col_range = [&](int c_lo, int c_n, int& b, int& e) {  // this warp's columns of [c_lo, c_lo + c_n)
        const int half = ((c_n / 2 + 15) / 16) * 16;
        b = c_lo + (ch ? min(half, c_n) : 0);
        e = c_lo + (ch ? c_n : min(half, c_n));
    };
    auto park = [&](float* dst, int c_lo, int c_n, uint32_t col0) {  // dst[(c - c_lo)][row] = accumulator
        int cb, ce;
        col_range(c_lo, c_n, cb, ce);
        for (int c0 = cb; c0 < ce; c0 += 16) {
            uint32_t v[16];
            if (live) tc_ld16(tmem + ((uint32_t)(lq * 32) << 16) + col0 + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                dst[(c0 - c_lo + j) * TC_BM + lq * 32 + lane] = live ? __uint_as_float(v[j]) : 0.f;
        }
    };
    if (p.splits == 1 && p.h) {
        // SwiGLU: the accumulator through shared memory (the stages are free), so
        // a thread sees both rows of a gate / up pair
        float* st = reinterpret_cast<float*>(smem);
        park(st, 0, p.NTp, 0u);
        __syncthreads();
        if (live) tc_swiglu_rows(p, st, 0, p.NTp, nb, tid);
    } else if (p.splits == 1) {
        if (live)
            for (int wj = 0; wj < wn; ++wj) {
                const int nw = n + wj * TC_BM;
                int cb, ce;
                col_range(0, p.NTp, cb, ce);
                for (int c0 = cb; c0 < ce; c0 += 16) {
                    uint32_t v[16];
                    tc_ld16(tmem + ((uint32_t)(lq * 32) << 16) + (uint32_t)(wj * 128 + c0), v);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < p.M && nw < p.N) tc_store(p, c0 + j, nw, __uint_as_float(v[j]));
                }
            }
    } else {
        // every MMA has completed and every stage has been read: the stages take the
        // accumulator, TC_RED_T token rows per pass.  Each CTA parks the pass's rows
        // (red[t][row]; zeros if this split has no K blocks or a wait ran out: the
        // status word says which), then hands every other split the rows that split
        // sums by one bulk copy into its receive buffer (rcv, one slot per sender),
        // and sums its own rows from its shared memory in split order.
        float* red = reinterpret_cast<float*>(smem);
        const int rows = min(p.NTp, TC_RED_T), per = rows / p.splits;
        float* rcv = red + (size_t)rows * TC_BM;
        volatile int* good_w = reinterpret_cast<volatile int*>(done + 1) + 2;
        if (tid == 0) *good_w = good ? 1 : 0;
        const uint32_t bytes_in = (uint32_t)((p.splits - 1) * per * TC_BM * 4);
        const bool vec = (p.ldo & 3) == 0 &&
                         ((reinterpret_cast<uintptr_t>(p.resid ? (const void*)p.resid : (const void*)p.out) & 15) == 0);
        bool all_good = true;
        for (int q = 0; q * TC_RED_T < p.NTp; ++q) {
            const int tq = q * TC_RED_T;
            park(red, 0, rows, (uint32_t)tq);
            fence_proxy_async_smem();
            if (tid == 0) mbar_arrive_expect_tx(rbar, bytes_in);
            cluster_sync_all();
            if (q == 0)  // thread r reads rank r's word: one remote round trip
                all_good = __syncthreads_and(tid >= p.splits ||
                                             ld_dsmem_s32(dsmem_addr((const void*)good_w, (uint32_t)tid)) != 0);
            if (!all_good) {  // every CTA of the cluster sees the same words and leaves here
                cluster_sync_all();  // (after every CTA has read them)
                break;
            }
            if (tid < p.splits && tid != sp) {
                const int slot = sp < tid ? sp : sp - 1;  // this CTA's slot in the receiver's buffer
                bulk_s2cluster(dsmem_addr(rcv + (size_t)slot * per * TC_BM, (uint32_t)tid),
                               red + (size_t)tid * per * TC_BM, (uint32_t)(per * TC_BM * 4),
                               dsmem_addr(rbar, (uint32_t)tid));
            }
            bool got = mbar_wait_bounded(rbar, (uint32_t)(q & 1), nullptr);
            if (!got && p.status) set_status(p.status, HGD_ERR_TIMEOUT);
            got = __syncthreads_and(got);
            if (got) {
                const int t_lo = sp * per, t_hi = min(t_lo + per, p.M - tq);
                switch (p.splits) {
                    case 2: tc_split_sum<2>(p, red, rcv, per, sp, t_lo, t_hi, tq, nb, tid, vec); break;
                    case 4: tc_split_sum<4>(p, red, rcv, per, sp, t_lo, t_hi, tq, nb, tid, vec); break;
                    default: tc_split_sum<8>(p, red, rcv, per, sp, t_lo, t_hi, tq, nb, tid, vec); break;
                }
                if (p.h) {
                    __syncthreads();
                    tc_swiglu_rows(p, red + (size_t)t_lo * TC_BM, tq + t_lo, tq + t_lo + per, nb, tid);
                }
            }
            // every copy of the pass has landed (each CTA waited for its own) before
            // red and rcv are written again, and before any CTA leaves; every CTA of
            // the cluster runs every pass, so the cluster barriers always match
            cluster_sync_all();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
    }
}

}  // namespace hgd
