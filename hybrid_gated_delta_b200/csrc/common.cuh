// common.cuh -- device helpers shared by the sm_100a kernels: bf16 bit
// conversions, PTX wrappers for mbarriers, bulk (TMA) copies and mma.sync, warp
// reductions, bounded waits and programmatic-dependent-launch controls.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hgd.h"

namespace hgd {

typedef uint16_t bf16_t;

// Limit of every in-kernel wait, in nanoseconds of %globaltimer.  A wait that
// runs out sets HGD_ERR_TIMEOUT in the status word and the kernel returns.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ float bf2f(bf16_t h) { return __uint_as_float(((uint32_t)h) << 16); }
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ bf16_t f2bf(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<bf16_t*>(&b);
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    return (uint32_t)f2bf(lo) | ((uint32_t)f2bf(hi) << 16);
}

__device__ __forceinline__ float silu_f(float t) { return t / (1.0f + expf(-t)); }
__device__ __forceinline__ float sigmoid_f(float t) { return 1.0f / (1.0f + expf(-t)); }
__device__ __forceinline__ float softplus_f(float t) {
    return fmaxf(t, 0.0f) + log1pf(expf(-fabsf(t)));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sums over the warp of N = 2, 4, 8, 16 or 32 values per lane (x[i] the lane's
// share of sum i), with warp_sum's pairings: level m pairs lane l with l ^ m
// (m = 16, 8, 4, 2, 1), so every total is bitwise warp_sum(x[i]).  At each level
// a lane keeps half of its running sums (the lower half where bit m of the lane
// is clear) and sends the other half, so the whole reduction takes about N - 1
// shuffles instead of 5 N.  Afterwards sum i sits in the lanes whose bits
// 4..(5 - log2 N) spell i from the top; returned is this lane's sum.
template <int N>
__device__ __forceinline__ float warp_sum_transposed(float (&x)[N], int lane) {
    static_assert(N == 2 || N == 4 || N == 8 || N == 16 || N == 32, "N");
#pragma unroll
    for (int m = 16, c = N; m >= 1 && c > 1; m >>= 1, c >>= 1) {
        const bool up = lane & m;
#pragma unroll
        for (int i = 0; i < c / 2; ++i) {
            const float keep = up ? x[i + c / 2] : x[i], send = up ? x[i] : x[i + c / 2];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
    }
    float v = x[0];
    // the levels below the last split: plain butterfly on the one sum left
#pragma unroll
    for (int m = 16 >> (N == 32 ? 5 : N == 16 ? 4 : N == 8 ? 3 : N == 4 ? 2 : 1); m >= 1; m >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, m);
    return v;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(int32_t* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ----------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase of `parity` to complete; false if the wait limit ran out
// or `abort_flag` (shared) was raised by another thread of the CTA.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort_flag && *abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
}

// As mbar_wait_bounded, sleeping `ns` nanoseconds between tests: for a waiter
// that is not on a critical path and should leave the issue slots of its SM
// sub-partition to the warps that are.
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                 unsigned ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        __nanosleep(ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (abort_flag && *abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
}

// ----------------------------------------------------------- bulk (TMA) copy
// 1-D bulk copy global -> shared, completing `bytes` of transaction count on
// `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.  The copy lands in
// this CTA's own shared memory only.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
// 16-byte asynchronous copy global -> shared (cp.async, L2 only), committed in
// groups; a thread waits for all but its newest group.
__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src_gmem) : "memory");
}
// 4-byte asynchronous copy global -> shared (cp.async.ca).
__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src_gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst_smem)), "l"(src_gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most the newest committed group of this thread is in flight.
__device__ __forceinline__ void cp_async_wait_prior() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// Prefetch of the line holding p into this SM's L1.
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned start) into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// --------------------------------------------------------------- shared loads
__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_addr(p)));
    return v;
}

// ---------------------------------------------------------------- mma.sync
// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One (row, head) of the gated RMSNorm by one warp: o row orow[d], z row
// zrow[d], gains w[d]; put(i, value) receives bf16(o r w silu(bf16(z))) with
// r = rsqrt(mean(o^2) + eps).  Shared by k_gated_norm and the GDN layer kernel's
// fused form, so both give the same bits.
template <class Put>
__device__ __forceinline__ void gated_norm_warp(const float* orow, const float* zrow, const bf16_t* w, int d,
                                                float eps, int lane, Put put) {
    auto emit = [&](int i, float ov, float zv, float wv, float r) {
        const float zb = bf2f(f2bf(zv));
        put(i, f2bf(ov * r * wv * silu_f(zb)));
    };
    // heads of up to GR * 32 values are read once, into registers
    constexpr int GR = 8;
    if (d <= GR * 32) {
        float ov[GR], zv[GR], wv[GR];  // o, z and the gains, loaded together
#pragma unroll
        for (int u = 0; u < GR; ++u)
            if (lane + 32 * u < d) {
                ov[u] = orow[lane + 32 * u];
                zv[u] = zrow[lane + 32 * u];
                wv[u] = bf2f(w[lane + 32 * u]);
            }
        float ss = 0.f;
#pragma unroll
        for (int u = 0; u < GR; ++u)
            if (lane + 32 * u < d) ss = fmaf(ov[u], ov[u], ss);
        ss = warp_sum(ss);
        const float r = rsqrtf(ss / (float)d + eps);
#pragma unroll
        for (int u = 0; u < GR; ++u)
            if (lane + 32 * u < d) emit(lane + 32 * u, ov[u], zv[u], wv[u], r);
        return;
    }
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) ss = fmaf(orow[i], orow[i], ss);
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)d + eps);
    for (int i = lane; i < d; i += 32) emit(i, orow[i], zrow[i], bf2f(w[i]), r);
}

// ------------------------------------------- tensor-core operand layout
// Token rows as the tensor-core GEMM (gemm_tc.cuh) reads them: per 64-wide k
// block a tile of NTp rows in 8 x 8 core matrices (8 rows of 16 bytes, 128
// contiguous bytes), core (row group g, k group j) at element (g * 8 + j) * 64.
// Element offset of X[t][k]; the 8 elements of an aligned k octet are contiguous.
constexpr int TC_BK = 64;  // k per block (and per GEMM pipeline stage)
__host__ __device__ inline size_t tc_x_elem(int t, int k, int NTp) {
    const int kk = k & (TC_BK - 1);
    return (size_t)(k >> 6) * NTp * TC_BK + (size_t)(((t >> 3) * 8 + (kk >> 3)) * 64 + (t & 7) * 8 + (kk & 7));
}

// Named barrier over the first `nthreads` threads of the CTA (id 1..15).
__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace hgd
