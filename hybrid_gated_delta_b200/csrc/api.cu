// api.cu -- extern "C" entry points of libhgd (declared in include/hgd.h):
// argument validation, launch planning and the per-layer launch sequence of the
// decode stack.  The library allocates no device memory; every buffer is the
// caller's.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <utility>
#include <cstdio>
#include <cmath>
#include <cstring>
#include <mutex>

#include "attn.cuh"
#include "common.cuh"
#include "gdn.cuh"
#include "gdn_chunk.cuh"
#include "tc_chain.cuh"
#include "gemv.cuh"
#include "gemm_tc.cuh"
#include "stack.cuh"

using namespace hgd;

namespace {

// ------------------------------------------------------------ context identity
// What the library caches per device (a kernel's shared-memory attribute, its
// occupancy, the device address of a built-in array) belongs to a CUDA context,
// not to the device ordinal: after a device reset the next call runs in a new
// context, where attributes are unset and a module variable may sit at another
// address.  Every such cache is therefore keyed on the current context's id
// (cuCtxGetId: unique within the process, never reused), read through the
// runtime's driver entry points so the library links no driver stub.
typedef int (*CtxGetCurrentFn)(void**);
typedef int (*CtxGetIdFn)(void*, unsigned long long*);

// Id of the calling thread's current context; 0 when there is none yet or the
// driver cannot tell (callers then cache nothing).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_cur = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();
    });
    if (!get_cur || !get_id) return 0;
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (get_cur(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0) return 0;
    return id;
}

// A value cached per context: a few slots, each holding (context id, value),
// read and written under one mutex.  Lookups from concurrent host threads are
// safe; a context that is not found is simply computed again.
template <typename V, int N = 8>
struct CtxCache {
    std::mutex mu;
    unsigned long long id[N] = {};
    V val[N] = {};
    int next = 0;
    bool get(unsigned long long ctx, V* out) {
        if (!ctx) return false;
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < N; ++i)
            if (id[i] == ctx) { *out = val[i]; return true; }
        return false;
    }
    void put(unsigned long long ctx, const V& v) {
        if (!ctx) return;
        std::lock_guard<std::mutex> g(mu);
        for (int i = 0; i < N; ++i)
            if (id[i] == ctx) { val[i] = v; return; }
        id[next] = ctx;
        val[next] = v;
        next = (next + 1) % N;
    }
};

// Sets the dynamic shared-memory limit of `kern` once per context.
template <typename K>
cudaError_t ensure_smem_attr(K kern, CtxCache<int>& done) {
    const unsigned long long ctx = current_ctx_id();
    int v = 0;
    if (done.get(ctx, &v)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GV_SMEM_LIMIT);
    if (e != cudaSuccess) return e;
    done.put(ctx, 1);
    return cudaSuccess;
}

// ------------------------------------------------------------ device info
struct DevInfo {
    int ok;    // 1 = sm_100, 0 = unsupported, -1 = cuda error
    int sms;
};

// The architecture and SM count of the current device (properties of the
// device, so cached per ordinal; packed in one atomic word: bit 31 set = known).
int device_info(DevInfo* di) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return HGD_ERR_CUDA; }
    static std::atomic<unsigned> cache[64];
    const bool cache_ok = dev >= 0 && dev < 64;
    const unsigned c = cache_ok ? cache[dev].load(std::memory_order_relaxed) : 0u;
    if (c & 0x80000000u) {
        *di = DevInfo{(int)((c >> 30) & 1u), (int)(c & 0xFFFFu)};
        return di->ok == 1 ? HGD_OK : HGD_ERR_UNSUPPORTED_DEVICE;
    }
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    DevInfo d{major == 10 ? 1 : 0, sms};
    if (cache_ok)
        cache[dev].store(0x80000000u | ((unsigned)d.ok << 30) | ((unsigned)sms & 0xFFFFu), std::memory_order_relaxed);
    *di = d;
    return d.ok == 1 ? HGD_OK : HGD_ERR_UNSUPPORTED_DEVICE;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status(cudaError_t e) {
    if (e == cudaSuccess) return HGD_OK;
    cudaGetLastError();
    return HGD_ERR_CUDA;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
// The same, with the grid in clusters of cluster_x consecutive CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ------------------------------------------------------------- GEMV plans
// Row blocks below this count use split slabs (partials through the workspace)
// when a workspace is given.  The arithmetic of every output is the same in both
// modes, so the threshold only moves work between warps.
constexpr int kSplitMaxRowblk = 2048;

struct GemvPlan {
    int nt, mchunk, x_bytes;
    size_t smem;
};

size_t gv_fixed_bytes(int mp) { return (size_t)GV_CW * mp * 8 + (size_t)GV_CW * GV_ROWS * mp * 4 + 16; }

bool plan_gemv(int M, int K, GemvPlan* pl) {
    const int want = (M + 7) / 8;
    int nt = want <= 1 ? 1 : (want <= 2 ? 2 : 4);
    for (; nt >= 1; nt >>= 1) {
        const int mp = 8 * nt;
        const int xb = gv_align16(mp * (K + GV_PAD) * 2);
        const size_t smem = xb + gv_fixed_bytes(mp);
        if (smem <= (size_t)GV_SMEM_LIMIT) {
            pl->nt = nt;
            pl->mchunk = mp;
            pl->x_bytes = xb;
            pl->smem = smem;
            return true;
        }
    }
    return false;
}

int rowblocks_of(int N, bool swiglu) { return swiglu ? (N + 7) / 8 : (N + GV_ROWS - 1) / GV_ROWS; }

// Workspace layout: the row-block counters at a fixed place (so that every GEMV
// sharing a workspace finds them at zero), then the slab partials.
constexpr size_t kWsCounterBytes = (size_t)kSplitMaxRowblk * 4;

// Workspace bytes a GEMV of this shape uses in split mode (0 if it never splits).
size_t gemv_ws_bytes(int M, int N, int K, bool swiglu) {
    GemvPlan pl;
    if (!plan_gemv(M, K, &pl)) return 0;
    const int nrb = rowblocks_of(N, swiglu);
    if (nrb >= kSplitMaxRowblk) return 0;
    return kWsCounterBytes + (size_t)nrb * gv_slabs(K) * GV_ROWS * pl.mchunk * 4;
}

// CTAs of one GEMV launch: one per work item up to as many as can be resident
// at once (the launch is one wave).
template <int NT, int PRO, int EPI>
cudaError_t launch_gemv_t(GemvParams p, size_t smem, int sms, cudaStream_t s, int* grid_out) {
    auto kern = k_gemv<NT, PRO, EPI>;
    static CtxCache<int> attr_done;
    struct Occ { int v[4]; };
    static CtxCache<Occ> occ_cache;
    cudaError_t e = ensure_smem_attr(kern, attr_done);
    if (e != cudaSuccess) return e;
    // occupancy for this shared-memory size (bucketed by 56 KB, cached per context)
    const unsigned long long ctx = current_ctx_id();
    const int bucket = std::min(3, (int)(smem / (56 * 1024)));
    Occ oc{};
    occ_cache.get(ctx, &oc);
    int occ = oc.v[bucket];
    if (occ == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, GV_THREADS, smem);
        if (e != cudaSuccess) return e;
        occ = std::max(1, occ);
        occ_cache.get(ctx, &oc);
        oc.v[bucket] = occ;
        occ_cache.put(ctx, oc);
    }
    // items go to CTAs first (slot = warp * grid + cta), so a GEMV with few items
    // still spreads over every SM
    const int grid = std::max(1, std::min(p.n_items, occ * sms));
    if (grid_out) *grid_out = grid;
    return launch_pdl(kern, dim3(grid), dim3(GV_THREADS), smem, s, p);
}

template <int PRO, int EPI>
cudaError_t launch_gemv_nt(int nt, const GemvParams& p, size_t smem, int sms, cudaStream_t s, int* grid_out) {
    switch (nt) {
        case 1: return launch_gemv_t<1, PRO, EPI>(p, smem, sms, s, grid_out);
        case 2: return launch_gemv_t<2, PRO, EPI>(p, smem, sms, s, grid_out);
        default: return launch_gemv_t<4, PRO, EPI>(p, smem, sms, s, grid_out);
    }
}

// Launch a GEMV over all M rows, in chunks of the plan's M tile (each chunk
// re-streams the weights; only very large M * K needs more than one).
template <int PRO, int EPI>
int run_gemv(GemvParams p, int M, int sms, void* ws, size_t ws_bytes, cudaStream_t s, int* grid_out = nullptr) {
    GemvPlan pl;
    if (!plan_gemv(M, p.K, &pl)) return HGD_ERR_UNSUPPORTED_SHAPE;
    p.nks = gv_slabs(p.K);
    p.n_rowblk = rowblocks_of(p.N, EPI == EPI_SWIGLU);
    p.x_bytes = pl.x_bytes;
    const size_t need = gemv_ws_bytes(M, p.N, p.K, EPI == EPI_SWIGLU);
    p.split = (EPI != EPI_ARGMAX && ws && need && ws_bytes >= need) ? 1 : 0;
    if (p.split) {
        p.ws_mp = pl.mchunk;
        p.ws_cnt = static_cast<int32_t*>(ws);
        p.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsCounterBytes);
    }
    p.n_items = p.n_rowblk * (p.split ? p.nks : 1);
    int grid = 0;
    for (int m0 = 0; m0 < M; m0 += pl.mchunk) {
        GemvParams q = p;
        q.M = std::min(pl.mchunk, M - m0);
        q.m0 = m0;
        if (q.x) q.x += m0 * q.x_ld;
        if (q.tokens) q.tokens += m0;
        if (q.resid_out) q.resid_out += m0 * q.resid_out_ld;
        if (q.o) q.o += m0 * q.o_ld;
        if (q.z) q.z += m0 * q.z_ld;
        if (q.resid) q.resid += m0 * q.resid_ld;
        if (q.rope_q) q.rope_q += (size_t)m0 * q.rope_nq * q.rope_hd;
        if (q.y) {
            const int es = (EPI == EPI_F32 || EPI == EPI_QKV_CONV || EPI == EPI_ROPE) ? 4 : 2;
            q.y = reinterpret_cast<uint8_t*>(q.y) + (size_t)m0 * q.y_ld * es;
        }
        if (q.logits) q.logits += m0 * q.logits_ld;
        // ARGMAX partials are [M][grid]; the grid is the same for every chunk
        if (q.best_v && m0) { q.best_v += (size_t)m0 * grid; q.best_i += (size_t)m0 * grid; }
        // (conv tails of streams in this chunk are updated in place; the next
        // chunk continues from them in stream order)
        cudaError_t e = launch_gemv_nt<PRO, EPI>(pl.nt, q, pl.smem, sms, s, &grid);
        if (e != cudaSuccess) return launch_status(e);
    }
    if (grid_out) *grid_out = grid;
    return HGD_OK;
}

int gemv_chunks(int M, int K) {
    GemvPlan pl;
    if (!plan_gemv(M, K, &pl)) return -1;
    return (M + pl.mchunk - 1) / pl.mchunk;
}

// ------------------------------------------------------------ stack layout
struct Dims {
    int L, D, V, H, dk, dv, kc, nq, nkv, hd, I, every;
    int Hk;       // GDN query/key heads; H is the value heads (a multiple of Hk)
    int untied;   // 1: the LM head is its own tensor (HGD_W_LM_HEAD)
    int n_gdn, n_attn;
    int64_t C, gdn_out, attn_out;
};

bool is_attn_layer(const hgd_config* c, int l) { return (l % c->attn_every) == c->attn_every - 1; }

int dims_of(const hgd_config* c, Dims* d) {
    if (!c) return HGD_ERR_INVALID_ARG;
    if (c->n_layers < 1 || c->n_layers > HGD_MAX_LAYERS || c->attn_every < 1) return HGD_ERR_INVALID_ARG;
    if (c->hidden < 32 || c->vocab < 1 || c->gdn_heads < 1 || c->mlp_inter < 1 || c->attn_q_heads < 1 ||
        c->attn_kv_heads < 1)
        return HGD_ERR_INVALID_ARG;
    if (c->gdn_v_heads < 0 || (c->gdn_v_heads > 0 && c->gdn_v_heads % c->gdn_heads != 0) ||
        (c->untied_head != 0 && c->untied_head != 1))
        return HGD_ERR_INVALID_ARG;
    d->L = c->n_layers; d->D = c->hidden; d->V = c->vocab;
    d->Hk = c->gdn_heads; d->H = c->gdn_v_heads > 0 ? c->gdn_v_heads : c->gdn_heads;
    d->untied = c->untied_head;
    d->dk = c->gdn_dk; d->dv = c->gdn_dv; d->kc = c->conv_k; d->nq = c->attn_q_heads;
    d->nkv = c->attn_kv_heads; d->hd = c->attn_head_dim; d->I = c->mlp_inter; d->every = c->attn_every;
    d->n_gdn = d->n_attn = 0;
    for (int l = 0; l < d->L; ++l) (is_attn_layer(c, l) ? d->n_attn : d->n_gdn)++;
    d->C = 2 * (int64_t)d->Hk * d->dk + (int64_t)d->H * d->dv;
    d->gdn_out = d->C + (int64_t)d->H * d->dv + 2 * d->H;
    d->attn_out = 2 * (int64_t)d->nq * d->hd + 2 * (int64_t)d->nkv * d->hd;
    return HGD_OK;
}

int check_supported(const Dims& d) {
    const bool ok =
        d.D % 32 == 0 && d.D <= 65536 && (d.H * d.dv) % 32 == 0 && (d.nq * d.hd) % 32 == 0 &&
        d.I % 32 == 0 && (d.dk == 32 || d.dk == 64 || d.dk == 128 || d.dk == 256) && d.dv % 16 == 0 &&
        d.dv <= 1024 && d.kc == 4 && (d.hd == 32 || d.hd == 64 || d.hd == 128 || d.hd == 256) &&
        d.nq % d.nkv == 0 &&
        d.nq / d.nkv <= ATTN_MAX_GROUP;
    return ok ? HGD_OK : HGD_ERR_UNSUPPORTED_SHAPE;
}

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

// base^(-2/hd): the RoPE frequency ratio between neighbouring dim pairs.
double rope_inv1_of(const Dims& d, float base) { return std::pow((double)base, -2.0 / (double)d.hd); }

// numel of one weight tensor (0 if absent)
size_t weight_numel(const Dims& d, const hgd_config* c, int layer, int t) {
    if (layer < 0) {
        if (t == HGD_W_EMBED) return (size_t)d.V * d.D;
        if (t == HGD_W_FINAL_NORM) return (size_t)d.D;
        if (t == HGD_W_LM_HEAD) return d.untied ? (size_t)d.V * d.D : 0;
        return 0;
    }
    const bool att = is_attn_layer(c, layer);
    switch (t) {
        case HGD_W_IN_NORM: case HGD_W_POST_NORM: return (size_t)d.D;
        case HGD_W_IN: return (size_t)(att ? d.attn_out : d.gdn_out) * d.D;
        case HGD_W_CONV: return att ? 0 : (size_t)d.C * d.kc;
        case HGD_W_A_LOG: case HGD_W_DT_BIAS: return att ? 0 : (size_t)d.H;
        case HGD_W_GNORM: return att ? 0 : (size_t)d.dv;
        case HGD_W_OUT: return (size_t)d.D * (att ? (size_t)d.nq * d.hd : (size_t)d.H * d.dv);
        case HGD_W_GATE: case HGD_W_UP: return (size_t)d.I * d.D;
        case HGD_W_DOWN: return (size_t)d.D * d.I;
        default: return 0;
    }
}

// How a tensor is stored: 0 plain, 1 packed matrix, 2 / 3 gate / up half of the
// packed SwiGLU region (which the gate tensor owns), 4 packed attention
// in-projection in rope_src_row's row order.  rows x cols is its logical shape
// for the packed kinds.
struct WeightKind { int kind; int64_t rows, cols; };

WeightKind weight_kind(const Dims& d, const hgd_config* c, int layer, int t) {
    if (layer < 0) {
        if (t == HGD_W_EMBED) return {1, d.V, d.D};
        if (t == HGD_W_LM_HEAD && d.untied) return {1, d.V, d.D};
        return {0, 0, 0};
    }
    const bool att = is_attn_layer(c, layer);
    switch (t) {
        case HGD_W_IN: return att ? WeightKind{4, d.attn_out, d.D} : WeightKind{1, d.gdn_out, d.D};
        case HGD_W_OUT: return {1, d.D, att ? (int64_t)d.nq * d.hd : (int64_t)d.H * d.dv};
        case HGD_W_GATE: return {2, d.I, d.D};
        case HGD_W_UP: return {3, d.I, d.D};
        case HGD_W_DOWN: return {1, d.D, d.I};
        default: return {0, 0, 0};
    }
}

// Bytes of the storage a tensor owns in the arena.
size_t weight_bytes(const Dims& d, const hgd_config* c, int layer, int t) {
    const WeightKind k = weight_kind(d, c, layer, t);
    switch (k.kind) {
        case 1: case 4: return (size_t)((k.rows + 15) / 16) * 16 * k.cols * 2;
        case 2: return (size_t)((k.rows + 7) / 8) * 16 * k.cols * 2;
        case 3: return 0;
        default: return weight_numel(d, c, layer, t) * 2;
    }
}

// Walk the arena in order; returns the total and, if (layer, t) matches, its offset.
size_t weight_walk(const Dims& d, const hgd_config* c, int want_layer, int want_t, size_t* off) {
    size_t pos = 0;
    const int glob[3] = {HGD_W_EMBED, HGD_W_FINAL_NORM, HGD_W_LM_HEAD};
    for (int g = 0; g < 3; ++g) {
        if (want_layer == -1 && want_t == glob[g] && off) *off = pos;
        pos += al256(weight_bytes(d, c, -1, glob[g]));
    }
    for (int l = 0; l < d.L; ++l) {
        size_t gate_off = 0;
        for (int t = 0; t < HGD_W_LAYER_COUNT; ++t) {
            if (t == HGD_W_GATE) gate_off = pos;
            if (l == want_layer && t == want_t && off) *off = (t == HGD_W_UP) ? gate_off : pos;
            pos += al256(weight_bytes(d, c, l, t));
        }
    }
    return pos;
}

enum ScratchIdx {
    SC_S = 0, SC_CONV, SC_KV, SC_POS, SC_RESID, SC_PROJ, SC_O, SC_QROT, SC_ATTN, SC_PART, SC_MLP,
    SC_BESTV, SC_BESTI, SC_WS, SC_BAR, SC_GN, SC_XN, SC_TCY, SC_TCLOG, SC_END, SC_COUNT
};
// The persistent launch's control region: control words, one 128-byte line per
// phase counter, then the phase timestamps.
constexpr size_t kBarCtrlBytes = (size_t)(SK_CTRL_WORDS + SK_MCNT_WORDS) * 4;
constexpr size_t kBarTraceOff = kBarCtrlBytes + (size_t)SK_MAX_PHASES * SK_CTR_STRIDE * 4;
#ifdef HGD_TRACE_DETAIL
// instrumented builds also keep every CTA's phase times after the timestamps
constexpr size_t kBarDetailOff = kBarTraceOff + (size_t)SK_TRACE_SLOTS * 8;
constexpr size_t kBarSlabOff = kBarDetailOff + (size_t)SK_MAX_PHASES * SK_TRACE_CTAS * 8 * 8;
constexpr size_t kBarBytes = kBarSlabOff + (size_t)SK_TRACE_SLABS * 4 * 8;
#else
constexpr size_t kBarBytes = kBarTraceOff + (size_t)SK_TRACE_SLOTS * 8;
#endif
constexpr int kBestG = 4096;  // max CTAs of the LM-head launch

int max_chunks_of(int Lmax) { return (Lmax + ATTN_CHUNK - 1) / ATTN_CHUNK; }

// A verify window's log (hgd_decode_layer_stack_verify): the copy of the conv
// tails the window runs on, then per GDN layer the rows' decay [B][T][H], write
// [B][T][H][dv], key [B][T][H][dk] and conv input [B][T][C] (fp32, each region
// 256-byte aligned).
struct VerifyLayout {
    size_t conv, alpha, delta, k, x, per_layer, first, total;
    size_t layer(int ig) const { return first + (size_t)ig * per_layer; }
};
VerifyLayout verify_layout(const Dims& d, int B, int T) {
    VerifyLayout v{};
    const size_t rows = (size_t)B * T;
    v.conv = 0;
    v.first = al256((size_t)d.n_gdn * B * (d.kc - 1) * d.C * 4);
    v.alpha = 0;
    v.delta = v.alpha + al256(rows * d.H * 4);
    v.k = v.delta + al256(rows * d.H * d.dv * 4);
    v.x = v.k + al256(rows * d.H * d.dk * 4);
    v.per_layer = v.x + al256(rows * d.C * 4);
    v.total = v.first + (size_t)d.n_gdn * v.per_layer;
    return v;
}

// keep's position advance: pos[b] += keep[b] for every stream whose count is in
// [0, T] (the others are reported and left).
__global__ void k_pos_keep(int32_t* pos, const int32_t* keep, int32_t* status, int B, int T) {
    pdl_launch();
    pdl_wait();
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int n = keep[b];
        if (n < 0 || n > T) set_status(status, HGD_ERR_INVALID_ARG);
        else pos[b] += n;
    }
}

// Split-K workspace of the stack: the largest any of its GEMVs uses at M rows.
struct TcPlan;
int64_t tc_rows128(int64_t n) { return (n + 127) / 128 * 128; }
int64_t tc_rows64(int64_t n) { return (n + 63) / 64 * 64; }

size_t stack_ws_bytes(const Dims& d, int M) {
    size_t w = 0;
    w = std::max(w, gemv_ws_bytes(M, (int)d.gdn_out, d.D, false));
    w = std::max(w, gemv_ws_bytes(M, (int)d.attn_out, d.D, false));
    w = std::max(w, gemv_ws_bytes(M, d.D, d.H * d.dv, false));
    w = std::max(w, gemv_ws_bytes(M, d.D, d.nq * d.hd, false));
    w = std::max(w, gemv_ws_bytes(M, d.I, d.D, true));
    w = std::max(w, gemv_ws_bytes(M, d.D, d.I, false));
    return w;
}

void state_layout(const Dims& d, int B, int Tmax, int Lmax, size_t* off) {
    const int64_t M = (int64_t)B * Tmax;
    size_t sz[SC_COUNT] = {};
    sz[SC_S] = (size_t)d.n_gdn * B * d.H * d.dv * d.dk * 4;
    sz[SC_CONV] = (size_t)d.n_gdn * B * (d.kc - 1) * d.C * 4;
    sz[SC_KV] = (size_t)d.n_attn * 2 * B * d.nkv * (size_t)Lmax * d.hd * 2;
    sz[SC_POS] = (size_t)B * 4;
    sz[SC_RESID] = (size_t)M * d.D * 2;
    sz[SC_PROJ] = (size_t)M * std::max(d.gdn_out, d.attn_out) * 4;
    sz[SC_O] = (size_t)M * d.H * d.dv * 4;
    sz[SC_QROT] = (size_t)M * d.nq * d.hd * 4;
    // (the tensor-core chain keeps these rows packed for its GEMMs: NTp rows)
    const size_t Mt = (size_t)std::max<int64_t>(M, tc_ntp((int)std::min<int64_t>(M, TC_MAXN)));
    sz[SC_ATTN] = Mt * d.nq * d.hd * 2;
    sz[SC_PART] = (size_t)M * d.nq * max_chunks_of(Lmax) * (d.hd + 2) * 4;
    sz[SC_MLP] = Mt * d.I * 2;
    sz[SC_BESTV] = (size_t)M * kBestG * 4;
    sz[SC_BESTI] = (size_t)M * kBestG * 4;
    sz[SC_WS] = stack_ws_bytes(d, (int)M);
    sz[SC_BAR] = kBarBytes;
    sz[SC_GN] = Mt * d.H * d.dv * 2;  // the chain's gated-norm rows for calls of many rows
    sz[SC_XN] = Mt * d.D * 2;         // the chain's RMSNorm rows for calls of many rows
    // the tensor-core chain: the head's argmax partials and its logits
    sz[SC_TCY] = (size_t)M * TC_AM_SLICES * 2 * 4;  // the head's argmax partials
    sz[SC_TCLOG] = (size_t)M * d.V * 4;
    size_t pos = 0;
    for (int i = 0; i < SC_END; ++i) { off[i] = pos; pos += al256(sz[i]); }
    off[SC_END] = pos;
}

int check_state_dims(int B, int Tmax, int Lmax) {
    if (B < 1 || Tmax < 1 || Lmax < 1) return HGD_ERR_INVALID_ARG;
    if ((int64_t)B * Tmax > 256 || Lmax > 16384) return HGD_ERR_UNSUPPORTED_SHAPE;
    return HGD_OK;
}

// ------------------------------------------------------- persistent launch
int sk_kmax(const Dims& d) { return std::max(std::max(d.D, d.H * d.dv), std::max(d.nq * d.hd, d.I)); }

constexpr int kSkPartialSlabs = 32;  // slab partials of the non-split phases' rounds

// Ring slots of the persistent launch for M token rows: the most (24, 16 or 8)
// that fit beside the token rows and the fixed buffers; 0 if none fits.
int sk_ring_slots(const Dims& d, int M) {
    for (int ns = 3 * SK_CW; ns >= SK_CW; ns -= SK_CW) {
        const size_t smem = (size_t)ns * SK_SLAB_BYTES + sk_fixed_bytes(M, sk_kmax(d), d.D, kSkPartialSlabs, ns);
        if (smem <= (size_t)GV_SMEM_LIMIT) return ns;
    }
    return 0;
}

size_t sk_smem_bytes(const Dims& d, int M, int ns) {
    return (size_t)ns * SK_SLAB_BYTES + sk_fixed_bytes(M, sk_kmax(d), d.D, kSkPartialSlabs, ns);
}

// The persistent launch covers calls of at most one MMA n-tile of token rows
// with a GDN key width of 64 or 128 and a shared-memory footprint that fits.
bool sk_supported(const Dims& d, int M) {
    return M <= SK_MAXM && (d.dk == 64 || d.dk == 128) && d.L * SK_PHASES_PER_LAYER + 2 <= SK_MAX_PHASES &&
           gv_slabs(sk_kmax(d)) <= kSkPartialSlabs && M * d.nq <= SK_MCNT_WORDS && sk_ring_slots(d, M) > 0;
}

template <int KPL, int DPL>
int sk_launch_t(const SkParams& prm, size_t smem, int sms, cudaStream_t s, bool launch, int occ_override) {
    auto kern = k_stack<KPL, DPL>;
    static CtxCache<int> attr_done;
    if (ensure_smem_attr(kern, attr_done) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    if (!launch) {
        // every CTA must be resident at once: the phases wait on one another
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, SK_THREADS, smem) != cudaSuccess) {
            cudaGetLastError();
            return HGD_ERR_CUDA;
        }
        if (occ_override >= 0) occ = occ_override;
        return occ < 1 ? HGD_ERR_NOT_CORESIDENT : HGD_OK;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sms);
    cfg.blockDim = dim3(SK_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return launch_status(cudaLaunchKernelEx(&cfg, kern, prm));
}

// The persistent kernel for this model's GDN key width (64 or 128) and
// attention head width (32, 64, 128 or 256).
// launch = false: only the co-residency check (occ_override >= 0 stands in for
// the occupancy the runtime reports); launch = true: the cooperative launch.
int sk_launch(const Dims& d, const SkParams& prm, size_t smem, int sms, cudaStream_t s, bool launch,
              int occ_override = -1) {
    if (d.dk == 128) {
        switch (d.hd) {
            case 256: return sk_launch_t<4, 8>(prm, smem, sms, s, launch, occ_override);
            case 128: return sk_launch_t<4, 4>(prm, smem, sms, s, launch, occ_override);
            case 64: return sk_launch_t<4, 2>(prm, smem, sms, s, launch, occ_override);
            default: return sk_launch_t<4, 1>(prm, smem, sms, s, launch, occ_override);
        }
    }
    switch (d.hd) {
        case 256: return sk_launch_t<2, 8>(prm, smem, sms, s, launch, occ_override);
        case 128: return sk_launch_t<2, 4>(prm, smem, sms, s, launch, occ_override);
        case 64: return sk_launch_t<2, 2>(prm, smem, sms, s, launch, occ_override);
        default: return sk_launch_t<2, 1>(prm, smem, sms, s, launch, occ_override);
    }
}

// ------------------------------------------------------- tensor-core GEMM plan
// A fixed function of (M, N, K): token rows padded to the MMA's N, 128-row
// weight tiles, a split of the K blocks that brings the CTA count near one wave
// (it depends on N and K only), as many shared-memory stages as fit.
struct TcPlan {
    int NTp, n_blocks, kb_per_split, splits, stages, wpb, npair, ctas;
    uint32_t tmem_cols;
    size_t xp_bytes;
};
// swiglu: the epilogue pairs gate and up rows through shared memory.
TcPlan tc_plan(int M, int N, int K, bool swiglu = false) {
    TcPlan q{};
    q.NTp = tc_ntp(M);
    q.n_blocks = tc_nblocks(N);
    const int nkb = K / TC_BK;
    // splits: a power of two up to a portable cluster, so the grid fills about
    // one wave of SMs; the last splits may get fewer K blocks (or none)
    const int want = std::max(1, std::min(std::min(nkb, TC_TARGET_CTAS / q.n_blocks), TC_MAX_SPLITS));
    q.splits = 1;
    while (q.splits * 2 <= want) q.splits *= 2;
    q.kb_per_split = (nkb + q.splits - 1) / q.splits;
    // many row blocks (the LM head): two weight blocks per CTA share each token
    // tile, so more of the bytes in flight are weights and the token rows are
    // re-read half as often (two CTAs of 2 x NTp TMEM columns fit an SM's 512)
    q.wpb = (q.splits == 1 && !swiglu && q.n_blocks >= 2 * TC_TARGET_CTAS && q.NTp <= 128) ? 2 : 1;
    // block pairs fill whole waves of two CTAs per SM; the remaining blocks run one
    // per CTA, so the last wave is made of half-length CTAs
    q.npair = q.wpb == 2 ? (q.n_blocks / 2) / (2 * TC_TARGET_CTAS) * (2 * TC_TARGET_CTAS) : 0;
    if (q.wpb == 2 && q.npair == 0) q.wpb = 1;
    q.ctas = q.wpb == 2 ? q.npair + (q.n_blocks - 2 * q.npair) : q.n_blocks * q.splits;
    const int ctas = q.ctas;
    // more than one wave of CTAs: stages for two CTAs per SM, so one's epilogue
    // overlaps the other's stream; otherwise every stage that fits
    const int per_sm = ctas > TC_TARGET_CTAS ? 2 : 1;
    const size_t avail = (size_t)GV_SMEM_LIMIT / per_sm - tc_smem_bytes(q.NTp, 0, q.wpb);
    q.stages = (int)std::min<size_t>(TC_MAX_STAGES, avail / tc_stage_bytes(q.NTp, q.wpb));
    if (q.stages < 2)
        q.stages = (int)std::min<size_t>(TC_MAX_STAGES, ((size_t)GV_SMEM_LIMIT - tc_smem_bytes(q.NTp, 0, q.wpb)) /
                                                            tc_stage_bytes(q.NTp, q.wpb));
    // with splits (or the SwiGLU pairing) the stages also hold the accumulator
    if (q.splits > 1 || swiglu) {
        const size_t bytes = q.splits > 1 ? tc_red_bytes(q.NTp, q.splits) : (size_t)q.NTp * TC_BM * 4;
        const int need = (int)((bytes + tc_stage_bytes(q.NTp) - 1) / tc_stage_bytes(q.NTp));
        q.stages = std::max(q.stages, need);
    }
    uint32_t c = 32;
    while ((int)c < (q.wpb - 1) * 128 + q.NTp) c <<= 1;  // weight block j at column j * 128
    q.tmem_cols = c;
    q.xp_bytes = ((size_t)q.NTp * K * 2 + 255) / 256 * 256;
    return q;
}
bool tc_shape_ok(int M, int N, int K) { return M >= 1 && M <= TC_MAXN && N >= 1 && K >= TC_BK && K % TC_BK == 0 && K <= 65536; }

// The tensor-core chain's packed weights, in one arena: the head, then per layer
// the in-projection, the out-projection, gate and up (one matrix: the gate rows,
// then the up rows from row tc_rows128(I)) and the down-projection; each in the
// GEMM's 128 x 64 core-matrix tiles, 256-byte aligned.  which: 0 in, 1 out,
// 2 gate+up, 3 down; layer -1: the head.
size_t tc_weight_bytes_of(int64_t N, int64_t K) { return al256((size_t)tc_rows128(N) * K * 2); }
size_t tc_walk(const Dims& d, const hgd_config* c, int want_layer, int want_which, size_t* off) {
    size_t pos = 0;
    if (want_layer == -1 && off) *off = pos;
    pos += tc_weight_bytes_of(d.V, d.D);
    for (int l = 0; l < d.L; ++l) {
        const bool att = is_attn_layer(c, l);
        const int64_t sh[4][2] = {{att ? d.attn_out : d.gdn_out, d.D},
                                  {d.D, att ? (int64_t)d.nq * d.hd : (int64_t)d.H * d.dv},
                                  {2 * tc_rows64(d.I), d.D},  // gate and up, interleaved by 64 rows
                                  {d.D, d.I}};
        for (int w = 0; w < 4; ++w) {
            if (l == want_layer && w == want_which && off) *off = pos;
            pos += tc_weight_bytes_of(sh[w][0], sh[w][1]);
        }
    }
    return pos;
}

// With resid set, the product is added to the bf16 rows resid[M][N] by the
// GEMM's epilogue instead of written to y.
// x_packed: x already holds the token rows in the GEMM's layout (tc_x_elem, NTp
// rows), and ws is not used.
// h (with I): the SwiGLU epilogue (W packed by k_tc_pack_w_swiglu, N = 2 *
// tc_rows64(I)); h receives bf16(silu(gate) * up) packed for the next GEMM.
int tc_run(const bf16_t* Wp, const bf16_t* x, int64_t x_ld, float* y, int M, int N, int K, void* ws,
           int32_t* status, cudaStream_t s, bf16_t* resid = nullptr, bool x_packed = false, bf16_t* h = nullptr,
           int I = 0) {
    const TcPlan q = tc_plan(M, N, K, h != nullptr);
    static CtxCache<int> attr_done;
    if (ensure_smem_attr(k_gemm_tc, attr_done) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    const bf16_t* Xp = x;
    cudaError_t e;
    if (!x_packed) {
        bf16_t* xp = static_cast<bf16_t*>(ws);
        const int chunks = q.NTp * (K / 8);
        e = launch_pdl(k_tc_pack_x, dim3(std::min(1184, (chunks + 255) / 256)), dim3(256), 0, s, x, x_ld, xp, M, K,
                       q.NTp);
        if (e != cudaSuccess) return launch_status(e);
        Xp = xp;
    }
    TcParams prm{};
    prm.Wp = Wp; prm.Xp = Xp; prm.out = y; prm.resid = resid; prm.h = h; prm.I = I; prm.status = status;
    prm.M = M; prm.N = N; prm.K = K; prm.NTp = q.NTp; prm.ldo = N;
    prm.n_blocks = q.n_blocks; prm.kb_per_split = q.kb_per_split; prm.splits = q.splits; prm.stages = q.stages;
    prm.wpb = q.wpb;
    prm.npair = q.npair;
    prm.tmem_cols = q.tmem_cols;
    const dim3 grid(q.ctas), block(TC_THREADS);
    const size_t smem = tc_smem_bytes(q.NTp, q.stages, q.wpb);
    e = q.splits > 1 ? launch_pdl_cluster(k_gemm_tc, grid, block, smem, s, q.splits, prm)
                     : launch_pdl(k_gemm_tc, grid, block, smem, s, prm);
    return launch_status(e);
}

// A wait that nothing completes: the bounded mbarrier wait of the slab rings and
// the tensor-core GEMM, on a barrier no thread arrives at.  It runs out after
// kWaitLimitNs and the kernel reports HGD_ERR_TIMEOUT in *status.
__global__ void k_check_bounded_wait(int32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0u, nullptr)) set_status(status, HGD_ERR_TIMEOUT);
}

// Diagnostic settings of one persistent launch (defaults: none).
struct SkDebug {
    unsigned long long wait_ns = kWaitLimitNs;
    int skip_cta = -1, skip_phase = -1;
};

// One call through the persistent launch: parameters, co-residency check, fresh
// control words, launch.  Nothing is enqueued if the check fails.
int sk_run(const hgd_model* m, const hgd_state* st, const Dims& d, const int32_t* tokens, int T, float* logits,
           int32_t* argmax, float* S_rec, float* tail_rec, int32_t* status_dev, cudaStream_t s,
           const SkDebug& dbg) {
    int rc;
    if (!al16(tokens) || !al16(argmax) || (logits && !al16(logits)) || (S_rec && !al16(S_rec)) ||
        (tail_rec && !al16(tail_rec)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    uint8_t* A = static_cast<uint8_t*>(st->arena);
    SkParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.L = d.L; prm.D = d.D; prm.V = d.V; prm.H = d.H; prm.dk = d.dk; prm.dv = d.dv; prm.nq = d.nq;
    prm.nkv = d.nkv; prm.hd = d.hd; prm.I = d.I; prm.every = d.every;
    prm.C = (int)d.C; prm.gdn_out = (int)d.gdn_out; prm.attn_out = (int)d.attn_out;
    prm.proj_ld = (int)std::max(d.gdn_out, d.attn_out); prm.kmax = sk_kmax(d);
    prm.eps = m->cfg.norm_eps; prm.rope_inv1 = rope_inv1_of(d, m->cfg.rope_base);
    prm.B = st->B; prm.T = T; prm.M = st->B * T; prm.Lmax = st->Lmax; prm.max_chunks = max_chunks_of(st->Lmax);
    prm.ns = sk_ring_slots(d, prm.M); prm.pb = kSkPartialSlabs;
    prm.embed = m->embed; prm.final_norm = m->final_norm;
    prm.head = m->lm_head ? m->lm_head : m->embed;
    prm.Hk = d.Hk;
    prm.S = reinterpret_cast<float*>(A + st->off[SC_S]);
    prm.conv = reinterpret_cast<float*>(A + st->off[SC_CONV]);
    prm.kv = reinterpret_cast<bf16_t*>(A + st->off[SC_KV]);
    prm.pos = reinterpret_cast<int32_t*>(A + st->off[SC_POS]);
    prm.resid = reinterpret_cast<bf16_t*>(A + st->off[SC_RESID]);
    prm.proj = reinterpret_cast<float*>(A + st->off[SC_PROJ]);
    prm.obuf = reinterpret_cast<float*>(A + st->off[SC_O]);
    prm.qrot = reinterpret_cast<float*>(A + st->off[SC_QROT]);
    prm.part = reinterpret_cast<float*>(A + st->off[SC_PART]);
    prm.mlp = reinterpret_cast<bf16_t*>(A + st->off[SC_MLP]);
    prm.attn = reinterpret_cast<bf16_t*>(A + st->off[SC_ATTN]);
    prm.bestv = reinterpret_cast<float*>(A + st->off[SC_BESTV]);
    prm.besti = reinterpret_cast<int32_t*>(A + st->off[SC_BESTI]);
    prm.tokens = tokens; prm.logits = logits; prm.argmax = argmax; prm.S_rec = S_rec; prm.tail_rec = tail_rec;
    prm.status = status_dev;
    prm.bar = reinterpret_cast<unsigned*>(A + st->off[SC_BAR]);
    prm.mcnt = prm.bar + SK_CTRL_WORDS;
    prm.trace = reinterpret_cast<unsigned long long*>(A + st->off[SC_BAR] + kBarTraceOff);
#ifdef HGD_TRACE_DETAIL
    prm.tdetail = reinterpret_cast<unsigned long long*>(A + st->off[SC_BAR] + kBarDetailOff);
    prm.tslab = reinterpret_cast<unsigned long long*>(A + st->off[SC_BAR] + kBarSlabOff);
#endif
    for (int l = 0; l < d.L; ++l)
        for (int t = 0; t < HGD_W_LAYER_COUNT; ++t) prm.layer[l].w[t] = m->w[l][t];
    prm.wait_ns = dbg.wait_ns;
    prm.dbg_skip_cta = dbg.skip_cta;
    prm.dbg_skip_phase = dbg.skip_phase;
    const size_t smem = sk_smem_bytes(d, prm.M, prm.ns);
    if ((rc = sk_launch(d, prm, smem, di.sms, s, false))) return rc;
    // fresh control words and phase counters for this call (an earlier call may
    // have stopped on a timeout)
    const size_t nph = (size_t)d.L * SK_PHASES_PER_LAYER + 2;
    if (cudaMemsetAsync(prm.bar, 0, kBarCtrlBytes + nph * SK_CTR_STRIDE * 4, s) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    return sk_launch(d, prm, smem, di.sms, s, true);
}

// The tensor-core chain's attention partials (k_attn_partial_tc), by head dim
// (one of 32, 64, 128, 256: check_supported admits no other).
template <int HD>
cudaError_t launch_attn_partial_tc_t(dim3 grid, cudaStream_t s, const AttnParams& a) {
    static CtxCache<int> attr_done;
    const cudaError_t e = ensure_smem_attr(k_attn_partial_tc<HD>, attr_done);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_attn_partial_tc<HD>, grid, dim3(256), attn_tc_smem_bytes(HD), s, a);
}
cudaError_t launch_attn_partial_tc(int hd, dim3 grid, cudaStream_t s, const AttnParams& a) {
    switch (hd) {
        case 256: return launch_attn_partial_tc_t<256>(grid, s, a);
        case 128: return launch_attn_partial_tc_t<128>(grid, s, a);
        case 64: return launch_attn_partial_tc_t<64>(grid, s, a);
        default: return launch_attn_partial_tc_t<32>(grid, s, a);
    }
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* hgd_status_string(int s) {
    switch (s) {
        case HGD_OK: return "ok";
        case HGD_ERR_INVALID_ARG: return "invalid argument";
        case HGD_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case HGD_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case HGD_ERR_CUDA: return "CUDA runtime error";
        case HGD_ERR_TIMEOUT: return "in-kernel wait timed out";
        case HGD_ERR_NOT_CORESIDENT: return "persistent launch cannot be co-resident";
        case HGD_ERR_NAN: return "NaN logit";
        case HGD_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
        case HGD_ERR_BUFFER_TOO_SMALL: return "arena smaller than required";
        default: return "unknown status";
    }
}

int hgd_version(void) { return 100; }

int hgd_gemv_workspace_bytes(int M, int N, int K, int swiglu, size_t* bytes) {
    if (!bytes || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (K % 32 != 0 || K > 65536) return HGD_ERR_UNSUPPORTED_SHAPE;
    *bytes = gemv_ws_bytes(M, N, K, swiglu != 0);
    return HGD_OK;
}

int hgd_gemv_bf16(const uint16_t* W, const uint16_t* x, void* y, int y_is_fp32, int M, int N, int K,
                  void* workspace, size_t workspace_bytes, hgd_stream_t stream) {
    if (!W || !x || !y || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (K % 32 != 0 || K > 65536) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W) || !al16(x) || !al16(y) || (workspace && !al16(workspace))) return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GemvParams p = {};
    p.W = W; p.N = N; p.K = K; p.x = x; p.x_ld = K; p.y = y; p.y_ld = N;
    if (y_is_fp32)
        return run_gemv<PRO_COPY, EPI_F32>(p, M, di.sms, workspace, workspace_bytes, (cudaStream_t)stream);
    return run_gemv<PRO_COPY, EPI_BF16>(p, M, di.sms, workspace, workspace_bytes, (cudaStream_t)stream);
}

int hgd_gemv_swiglu_bf16(const uint16_t* W_gate, const uint16_t* W_up, const uint16_t* x, uint16_t* h,
                         int M, int I, int K, void* workspace, size_t workspace_bytes, hgd_stream_t stream) {
    if (!W_gate || !W_up || !x || !h || M < 1 || I < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (K % 32 != 0 || K > 65536) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W_gate) || !al16(W_up) || !al16(x) || !al16(h) || (workspace && !al16(workspace)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GemvParams p = {};
    p.W = W_gate; p.W2 = W_up; p.N = I; p.K = K; p.x = x; p.x_ld = K; p.y = h; p.y_ld = I;
    return run_gemv<PRO_COPY, EPI_SWIGLU>(p, M, di.sms, workspace, workspace_bytes, (cudaStream_t)stream);
}

int hgd_check_bounded_wait(int32_t* status, hgd_stream_t stream) {
    if (!status) return HGD_ERR_INVALID_ARG;
    if (!al16(status)) return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    k_check_bounded_wait<<<1, 32, 0, (cudaStream_t)stream>>>(status);
    return launch_status(cudaGetLastError());
}

int hgd_gemm_tc_weight_bytes(int N, int K, size_t* bytes) {
    if (!bytes || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (!tc_shape_ok(1, N, K)) return HGD_ERR_UNSUPPORTED_SHAPE;
    *bytes = (size_t)tc_nblocks(N) * TC_BM * K * 2;
    return HGD_OK;
}

int hgd_gemm_tc_pack_weight(const uint16_t* W, uint16_t* Wp, int N, int K, hgd_stream_t stream) {
    if (!W || !Wp || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (!tc_shape_ok(1, N, K)) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W) || !al16(Wp)) return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    const int64_t chunks = (int64_t)tc_nblocks(N) * TC_BM * (K / 8);
    k_tc_pack_w<<<(unsigned)std::min<int64_t>(4736, (chunks + 255) / 256), 256, 0, (cudaStream_t)stream>>>(W, Wp, N, K);
    return launch_status(cudaGetLastError());
}

int hgd_gemm_tc_workspace_bytes(int M, int N, int K, size_t* bytes) {
    if (!bytes || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (!tc_shape_ok(M, N, K)) return HGD_ERR_UNSUPPORTED_SHAPE;
    const TcPlan q = tc_plan(M, N, K);
    *bytes = q.xp_bytes;
    return HGD_OK;
}

int hgd_gemm_tc_plan(int M, int N, int K, int* splits, int* stages) {
    if (!splits || !stages || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (!tc_shape_ok(M, N, K)) return HGD_ERR_UNSUPPORTED_SHAPE;
    const TcPlan q = tc_plan(M, N, K);
    *splits = q.splits;
    *stages = q.stages;
    return HGD_OK;
}

int hgd_gemm_tc_bf16(const uint16_t* Wp, const uint16_t* x, float* y, int M, int N, int K, void* workspace,
                     size_t workspace_bytes, int32_t* status, hgd_stream_t stream) {
    if (!Wp || !x || !y || !workspace || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (!tc_shape_ok(M, N, K)) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(Wp) || !al16(x) || !al16(y) || !al16(workspace)) return HGD_ERR_MISALIGNED;
    const TcPlan q = tc_plan(M, N, K);
    if (workspace_bytes < q.xp_bytes) return HGD_ERR_BUFFER_TOO_SMALL;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return tc_run(reinterpret_cast<const bf16_t*>(Wp), reinterpret_cast<const bf16_t*>(x), K, y, M, N, K, workspace,
                  status, (cudaStream_t)stream);
}

int hgd_conv1d_tail_update(const float* x, float* tail, const uint16_t* w, float* y, float* tail_rec,
                           int B, int T, int C, int kc, int apply_silu, hgd_stream_t stream) {
    if (!x || !tail || !w || !y || B < 1 || T < 1 || C < 1) return HGD_ERR_INVALID_ARG;
    if (kc < 2 || kc > 8) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(x) || !al16(tail) || !al16(w) || !al16(y) || (tail_rec && !al16(tail_rec)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    ConvParams p{x, tail, w, y, tail_rec, B, T, C, kc, apply_silu ? 1 : 0};
    const int64_t n = (int64_t)B * C;
    const int blocks = (int)((n + 255) / 256);
    return launch_status(launch_pdl(k_conv_tail, dim3(blocks), dim3(256), 0, (cudaStream_t)stream, p));
}

int hgd_gdn_decode_step(const float* q, const float* k, const float* v, int64_t row_stride, const float* g,
                        const float* b, float* S, float* o, uint16_t* o_bf16, float* S_rec, int B, int T,
                        int H, int dk, int dv, int l2norm_qk, hgd_stream_t stream) {
    return hgd_gdn_decode_step_grouped(q, k, v, row_stride, g, b, S, o, o_bf16, S_rec, B, T, H, H, dk, dv,
                                       l2norm_qk, stream);
}

int hgd_gdn_decode_step_grouped(const float* q, const float* k, const float* v, int64_t row_stride,
                                const float* g, const float* b, float* S, float* o, uint16_t* o_bf16,
                                float* S_rec, int B, int T, int Hk, int H, int dk, int dv, int l2norm_qk,
                                hgd_stream_t stream) {
    if (!q || !k || !v || !g || !b || !S || !o || B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1 || Hk < 1 ||
        H % Hk != 0)
        return HGD_ERR_INVALID_ARG;
    if (!(dk == 32 || dk == 64 || dk == 128 || dk == 256) || dv % GDN_ROWS != 0 || dv > 1024)
        return HGD_ERR_UNSUPPORTED_SHAPE;
    if (row_stride < (int64_t)Hk * dk || row_stride < (int64_t)H * dv) return HGD_ERR_INVALID_ARG;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(g) || !al16(b) || !al16(S) || !al16(o) ||
        (o_bf16 && !al16(o_bf16)) || (S_rec && !al16(S_rec)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GdnParams p{q, k, v, row_stride, g, b, S, o, o_bf16, S_rec, B, T, H, dk, dv, l2norm_qk ? 1 : 0, H / Hk};
    const dim3 grid(B * H, dv / GDN_ROWS), block(GDN_WARPS * 32);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (dk) {
        case 32: e = launch_pdl(k_gdn_step<1>, grid, block, 0, s, p); break;
        case 64: e = launch_pdl(k_gdn_step<2>, grid, block, 0, s, p); break;
        case 128: e = launch_pdl(k_gdn_step<4>, grid, block, 0, s, p); break;
        default: e = launch_pdl(k_gdn_step<8>, grid, block, 0, s, p); break;
    }
    return launch_status(e);
}

int hgd_gdn_prefill(const float* q, const float* k, const float* v, int64_t row_stride, const float* g,
                    const float* b, float* S, float* o, int B, int T, int H, int dk, int dv, int l2norm_qk,
                    hgd_stream_t stream) {
    if (!q || !k || !v || !g || !b || !S || !o || B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1)
        return HGD_ERR_INVALID_ARG;
    if (!(dk == 64 || dk == 128) || dv % GCK_DVB != 0 || dv > 1024) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (row_stride < (int64_t)H * dk || row_stride < (int64_t)H * dv) return HGD_ERR_INVALID_ARG;
    if (row_stride % 4 != 0) return HGD_ERR_MISALIGNED;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(g) || !al16(b) || !al16(S) || !al16(o))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GdnChunkParams p{q, k, v, row_stride, g, b, S, o, B, T, H, dv, l2norm_qk ? 1 : 0};
    const dim3 grid(B * H, dv / GCK_DVB), block(GCK_THREADS);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (dk == 128) {
        static CtxCache<int> attr;
        const int smem = (int)sizeof(GckSmem<128>);
        e = ensure_smem_attr(k_gdn_chunked<128>, attr);
        if (e == cudaSuccess) e = launch_pdl(k_gdn_chunked<128>, grid, block, smem, s, p);
    } else {
        static CtxCache<int> attr;
        const int smem = (int)sizeof(GckSmem<64>);
        e = ensure_smem_attr(k_gdn_chunked<64>, attr);
        if (e == cudaSuccess) e = launch_pdl(k_gdn_chunked<64>, grid, block, smem, s, p);
    }
    return launch_status(e);
}

// ------------------------------------------------- recurrence logs, keep

int hgd_gdn_window_log(const float* q, const float* k, const float* v, int64_t row_stride, const float* g,
                       const float* b, const float* S, float* o, uint16_t* o_bf16, float* log_alpha,
                       float* log_delta, float* log_k, int B, int T, int H, int dk, int dv, int l2norm_qk,
                       hgd_stream_t stream) {
    if (!q || !k || !v || !g || !b || !S || !o || !log_alpha || !log_delta || !log_k || B < 1 || T < 1 ||
        H < 1 || dk < 1 || dv < 1)
        return HGD_ERR_INVALID_ARG;
    if (!(dk == 32 || dk == 64 || dk == 128 || dk == 256) || dv % GDN_ROWS != 0 || dv > 1024)
        return HGD_ERR_UNSUPPORTED_SHAPE;
    if (row_stride < (int64_t)H * dk || row_stride < (int64_t)H * dv) return HGD_ERR_INVALID_ARG;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(g) || !al16(b) || !al16(S) || !al16(o) ||
        (o_bf16 && !al16(o_bf16)) || !al16(log_alpha) || !al16(log_delta) || !al16(log_k))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GdnLogParams p{q, k, v, row_stride, g, b, S, o, o_bf16, log_alpha, log_delta, log_k,
                   B, T, H, dk, dv, l2norm_qk ? 1 : 0, 1};
    const dim3 grid(B * H, dv / GDN_ROWS), block(GDN_WARPS * 32);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (dk) {
        case 32: e = launch_pdl(k_gdn_window_log<1>, grid, block, 0, s, p); break;
        case 64: e = launch_pdl(k_gdn_window_log<2>, grid, block, 0, s, p); break;
        case 128: e = launch_pdl(k_gdn_window_log<4>, grid, block, 0, s, p); break;
        default: e = launch_pdl(k_gdn_window_log<8>, grid, block, 0, s, p); break;
    }
    return launch_status(e);
}

int hgd_gdn_keep(float* S, const float* log_alpha, const float* log_delta, const float* log_k,
                 const int32_t* keep, int32_t* status_dev, int B, int T, int H, int dk, int dv, hgd_stream_t stream) {
    if (!S || !log_alpha || !log_delta || !log_k || !keep || B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1)
        return HGD_ERR_INVALID_ARG;
    if (!(dk == 32 || dk == 64 || dk == 128 || dk == 256) || dv % GDN_ROWS != 0 || dv > 1024)
        return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(S) || !al16(log_alpha) || !al16(log_delta) || !al16(log_k) || !al16(keep) ||
        (status_dev && !al16(status_dev)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    GdnKeepParams p{S, log_alpha, log_delta, log_k, keep, status_dev, B, T, H, dv};
    const dim3 grid(B * H, dv / GDN_ROWS), block(GDN_WARPS * 32);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    switch (dk) {
        case 32: e = launch_pdl(k_gdn_keep<1>, grid, block, 0, s, p); break;
        case 64: e = launch_pdl(k_gdn_keep<2>, grid, block, 0, s, p); break;
        case 128: e = launch_pdl(k_gdn_keep<4>, grid, block, 0, s, p); break;
        default: e = launch_pdl(k_gdn_keep<8>, grid, block, 0, s, p); break;
    }
    return launch_status(e);
}

int hgd_conv1d_keep(float* tail, const float* x, const int32_t* keep, int32_t* status_dev, int B, int T, int C,
                    int kc, hgd_stream_t stream) {
    if (!tail || !x || !keep || B < 1 || T < 1 || C < 1) return HGD_ERR_INVALID_ARG;
    if (kc < 2 || kc > 8) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(tail) || !al16(x) || !al16(keep) || (status_dev && !al16(status_dev))) return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    ConvKeepParams p{tail, x, keep, status_dev, B, T, C, kc};
    const int64_t n = (int64_t)B * C;
    return launch_status(launch_pdl(k_conv_keep, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                                    (cudaStream_t)stream, p));
}

// ---------------------------------------------------------------- stack

int hgd_model_arena_bytes(const hgd_config* cfg, size_t* bytes) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if (!bytes) return HGD_ERR_INVALID_ARG;
    *bytes = weight_walk(d, cfg, -2, -2, nullptr);
    return HGD_OK;
}

int hgd_model_tensor(const hgd_config* cfg, int layer, int tensor, size_t* offset, size_t* numel) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if (!offset || !numel) return HGD_ERR_INVALID_ARG;
    if (layer < -1 || layer >= d.L) return HGD_ERR_INVALID_ARG;
    if (layer == -1 && tensor != HGD_W_EMBED && tensor != HGD_W_FINAL_NORM && tensor != HGD_W_LM_HEAD)
        return HGD_ERR_INVALID_ARG;
    if (layer >= 0 && (tensor < 0 || tensor >= HGD_W_LAYER_COUNT)) return HGD_ERR_INVALID_ARG;
    size_t off = 0;
    weight_walk(d, cfg, layer, tensor, &off);
    *offset = off;
    *numel = weight_numel(d, cfg, layer, tensor);
    return HGD_OK;
}

int hgd_model_load_tensor(const hgd_config* cfg, void* arena, size_t arena_bytes, int layer, int tensor,
                          const uint16_t* src, hgd_stream_t stream) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (!arena || !src) return HGD_ERR_INVALID_ARG;
    if (layer < -1 || layer >= d.L) return HGD_ERR_INVALID_ARG;
    if (layer == -1 && tensor != HGD_W_EMBED && tensor != HGD_W_FINAL_NORM && tensor != HGD_W_LM_HEAD)
        return HGD_ERR_INVALID_ARG;
    if (layer >= 0 && (tensor < 0 || tensor >= HGD_W_LAYER_COUNT)) return HGD_ERR_INVALID_ARG;
    const size_t n = weight_numel(d, cfg, layer, tensor);
    if (n == 0) return HGD_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(arena) & 255u) || !al16(src)) return HGD_ERR_MISALIGNED;
    const size_t need = weight_walk(d, cfg, -2, -2, nullptr);
    if (arena_bytes < need) return HGD_ERR_BUFFER_TOO_SMALL;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    size_t off = 0;
    weight_walk(d, cfg, layer, tensor, &off);
    bf16_t* dst = reinterpret_cast<bf16_t*>(static_cast<uint8_t*>(arena) + off);
    const WeightKind k = weight_kind(d, cfg, layer, tensor);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (k.kind == 0) {
        const int blocks = (int)std::min<int64_t>(((int64_t)n + 255) / 256, 4096);
        e = launch_pdl(k_copy_u16, dim3(blocks), dim3(256), 0, s, (const bf16_t*)src, dst, (int64_t)n);
    } else {
        const int nrb = (k.kind == 1 || k.kind == 4) ? (int)((k.rows + 15) / 16) : (int)((k.rows + 7) / 8);
        const int64_t chunks = (int64_t)nrb * (k.cols / 32) * 64;
        const int blocks = (int)std::min<int64_t>((chunks + 255) / 256, 8192);
        const int mode = k.kind == 1 ? 0 : k.kind == 2 ? 1 : k.kind == 3 ? 2 : 3;
        e = launch_pdl(k_pack_weight, dim3(blocks), dim3(256), 0, s, (const bf16_t*)src, dst, (int)k.rows,
                       (int)k.cols, nrb, mode, d.nq, d.nkv, d.hd);
    }
    return launch_status(e);
}

int hgd_model_init(hgd_model* m, const hgd_config* cfg, const void* arena, size_t bytes) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (!m || !arena) return HGD_ERR_INVALID_ARG;
    if (!al16(arena) || (reinterpret_cast<uintptr_t>(arena) & 255u)) return HGD_ERR_MISALIGNED;
    const size_t need = weight_walk(d, cfg, -2, -2, nullptr);
    if (bytes < need) return HGD_ERR_BUFFER_TOO_SMALL;
    std::memset(m, 0, sizeof(*m));
    m->cfg = *cfg;
    const uint8_t* base = static_cast<const uint8_t*>(arena);
    size_t off = 0;
    weight_walk(d, cfg, -1, HGD_W_EMBED, &off);
    m->embed = reinterpret_cast<const uint16_t*>(base + off);
    weight_walk(d, cfg, -1, HGD_W_FINAL_NORM, &off);
    m->final_norm = reinterpret_cast<const uint16_t*>(base + off);
    if (d.untied) {
        weight_walk(d, cfg, -1, HGD_W_LM_HEAD, &off);
        m->lm_head = reinterpret_cast<const uint16_t*>(base + off);
    }
    for (int l = 0; l < d.L; ++l)
        for (int t = 0; t < HGD_W_LAYER_COUNT; ++t) {
            if (!weight_numel(d, cfg, l, t)) continue;
            weight_walk(d, cfg, l, t, &off);
            m->w[l][t] = reinterpret_cast<const uint16_t*>(base + off);
        }
    m->arena_bytes = need;
    return HGD_OK;
}

int hgd_state_arena_bytes(const hgd_config* cfg, int B, int Tmax, int Lmax, size_t* bytes) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if ((rc = check_state_dims(B, Tmax, Lmax))) return rc;
    if (!bytes) return HGD_ERR_INVALID_ARG;
    size_t off[SC_COUNT];
    state_layout(d, B, Tmax, Lmax, off);
    *bytes = off[SC_END];
    return HGD_OK;
}

int hgd_state_tensor(const hgd_config* cfg, int B, int Tmax, int Lmax, int tensor, size_t* offset,
                     size_t* numel) {
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if ((rc = check_state_dims(B, Tmax, Lmax))) return rc;
    if (!offset || !numel || tensor < 0 || tensor >= HGD_S_COUNT) return HGD_ERR_INVALID_ARG;
    size_t off[SC_COUNT];
    state_layout(d, B, Tmax, Lmax, off);
    *offset = off[tensor];
    switch (tensor) {
        case HGD_S_GDN: *numel = (size_t)d.n_gdn * B * d.H * d.dv * d.dk; break;
        case HGD_S_CONV: *numel = (size_t)d.n_gdn * B * (d.kc - 1) * d.C; break;
        case HGD_S_KV: *numel = (size_t)d.n_attn * 2 * B * d.nkv * (size_t)Lmax * d.hd; break;
        case HGD_S_RESID: *numel = (size_t)B * Tmax * d.D; break;
        default: *numel = (size_t)B; break;
    }
    return HGD_OK;
}

int hgd_state_init(hgd_state* st, const hgd_model* m, int B, int Tmax, int Lmax, void* arena, size_t bytes) {
    if (!st || !m || !arena) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_state_dims(B, Tmax, Lmax))) return rc;
    if (reinterpret_cast<uintptr_t>(arena) & 255u) return HGD_ERR_MISALIGNED;
    size_t off[SC_COUNT];
    state_layout(d, B, Tmax, Lmax, off);
    if (bytes < off[SC_END]) return HGD_ERR_BUFFER_TOO_SMALL;
    std::memset(st, 0, sizeof(*st));
    st->B = B; st->Tmax = Tmax; st->Lmax = Lmax;
    st->arena = arena;
    st->arena_bytes = off[SC_END];
    for (int i = 0; i < SC_COUNT && i < 32; ++i) st->off[i] = off[i];
    return HGD_OK;
}

int hgd_decode_layer_stack_launches(const hgd_model* m, int B, int T) {
    if (!m || B < 1 || T < 1) return -1;
    Dims d;
    if (dims_of(&m->cfg, &d)) return -1;
    const int M = B * T;
    if (sk_supported(d, M)) return 1;  // one cooperative launch (plus a barrier reset)
    int n = 0;
    for (int l = 0; l < d.L; ++l) {
        const bool att = is_attn_layer(&m->cfg, l);
        n += gemv_chunks(M, d.D);                                   // in-projection
        n += att ? 2 : 1;                                           // partial/merge or GDN mixer
        n += gemv_chunks(M, att ? d.nq * d.hd : d.H * d.dv);        // out-projection
        if (M > SK_MAXM) n += att ? 2 : 3;                          // norms once per row (in, gated, post)
        n += gemv_chunks(M, d.D) + gemv_chunks(M, d.I);             // SwiGLU, down
    }
    n += gemv_chunks(M, d.D) + 1;                                   // LM head, argmax
    if (M > SK_MAXM) n += 1;                                        // its norm, once per row
    return n;
}

int hgd_decode_layer_stack(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T, float* logits,
                           int32_t* argmax, float* S_rec, float* tail_rec, int32_t* status_dev,
                           hgd_stream_t stream) {
    if (!m || !st || !st->arena || !tokens || !argmax) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (!sk_supported(d, st->B * T))
        return hgd_decode_layer_stack_range(m, st, tokens, T, 0, m->cfg.n_layers, 1, logits, argmax, S_rec,
                                            tail_rec, status_dev, stream);
    return sk_run(m, st, d, tokens, T, logits, argmax, S_rec, tail_rec, status_dev, (cudaStream_t)stream,
                  SkDebug{});
}

int hgd_check_stack_timeout(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T,
                            int32_t* argmax, int skip_cta, int skip_phase, int wait_ms, int32_t* status_dev,
                            uint32_t* report_dev, hgd_stream_t stream) {
    if (!m || !st || !st->arena || !tokens || !argmax || !status_dev) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax || skip_cta < 0 || skip_phase < 0 || wait_ms < 1 || wait_ms > 2000)
        return HGD_ERR_INVALID_ARG;
    if (report_dev && !al16(report_dev)) return HGD_ERR_MISALIGNED;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (!sk_supported(d, st->B * T)) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (skip_phase > d.L * SK_PHASES_PER_LAYER) return HGD_ERR_INVALID_ARG;  // the LM head phase at most
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    if (skip_cta >= di.sms) return HGD_ERR_INVALID_ARG;
    SkDebug dbg;
    dbg.wait_ns = (unsigned long long)wait_ms * 1000000ull;
    dbg.skip_cta = skip_cta;
    dbg.skip_phase = skip_phase;
    cudaStream_t s = (cudaStream_t)stream;
    rc = sk_run(m, st, d, tokens, T, nullptr, argmax, nullptr, nullptr, status_dev, s, dbg);
    if (rc || !report_dev) return rc;
    // what ran out first, its phase and its CTA: control words 1..3
    const uint8_t* A = static_cast<const uint8_t*>(st->arena);
    if (cudaMemsetAsync(report_dev, 0, 16, s) != cudaSuccess ||
        cudaMemcpyAsync(report_dev, A + st->off[SC_BAR] + 4, 12, cudaMemcpyDeviceToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    return HGD_OK;
}

int hgd_check_not_coresident(const hgd_model* m, const hgd_state* st, int T) {
    if (!m || !st || !st->arena) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (!sk_supported(d, st->B * T)) return HGD_ERR_UNSUPPORTED_SHAPE;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    const int M = st->B * T;
    SkParams prm;
    std::memset(&prm, 0, sizeof(prm));
    return sk_launch(d, prm, sk_smem_bytes(d, M, sk_ring_slots(d, M)), di.sms, nullptr, false, 0);
}

// dv of the GDN layer kernel's fused gated-norm form (16 warps x 8 rows: a head per CTA).
constexpr int GDN_FUSED_DV = 128;
static_assert(GDN_CONV_K == GV_CONV_K, "one conv width");

// The GDN layer kernel over B streams: 8 state rows per warp where dv allows
// (32 rows per CTA), else 4; either way each row's arithmetic is the same.
cudaError_t launch_gdn_layer(const Dims& d, int B, const GdnLayerParams& g, cudaStream_t s) {
    const dim3 block(GDN_WARPS * 32);
    if (d.dv % (GDN_WARPS * 8) == 0) {
        const dim3 grid(B * d.H, d.dv / (GDN_WARPS * 8));
        switch (d.dk) {
            case 32: return launch_pdl(k_gdn_layer<1, 8>, grid, block, 0, s, g);
            case 64: return launch_pdl(k_gdn_layer<2, 8>, grid, block, 0, s, g);
            case 128: return launch_pdl(k_gdn_layer<4, 8>, grid, block, 0, s, g);
            default: return launch_pdl(k_gdn_layer<8, 8>, grid, block, 0, s, g);
        }
    }
    const dim3 grid(B * d.H, d.dv / GDN_ROWS);
    switch (d.dk) {
        case 32: return launch_pdl(k_gdn_layer<1, GDN_RPW>, grid, block, 0, s, g);
        case 64: return launch_pdl(k_gdn_layer<2, GDN_RPW>, grid, block, 0, s, g);
        case 128: return launch_pdl(k_gdn_layer<4, GDN_RPW>, grid, block, 0, s, g);
        default: return launch_pdl(k_gdn_layer<8, GDN_RPW>, grid, block, 0, s, g);
    }
}

// The kernel chain of layers [layer_begin, layer_end) and, if run_head, the head.
// With vl (a verify window): the conv runs on the log's copy of the tails and
// logs each row's conv input, the GDN layers log (alpha, delta, k) instead of
// writing the state, and the head leaves the positions as they are.
static int chain_run(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T, int layer_begin,
                     int layer_end, int run_head, float* logits, int32_t* argmax, float* S_rec, float* tail_rec,
                     int32_t* status_dev, hgd_stream_t stream, uint8_t* vl) {
    if (!m || !st || !st->arena) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if (layer_begin < 0 || layer_end > d.L || layer_begin > layer_end) return HGD_ERR_INVALID_ARG;
    if (layer_begin == 0 && layer_end > 0 && !tokens) return HGD_ERR_INVALID_ARG;
    if (run_head && !argmax) return HGD_ERR_INVALID_ARG;
    if ((tokens && !al16(tokens)) || (argmax && !al16(argmax))) return HGD_ERR_MISALIGNED;
    if ((rc = check_supported(d))) return rc;
    if ((logits && !al16(logits)) || (S_rec && !al16(S_rec)) || (tail_rec && !al16(tail_rec)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    const int B = st->B, M = B * T, Lmax = st->Lmax;
    uint8_t* A = static_cast<uint8_t*>(st->arena);
    float* Sall = reinterpret_cast<float*>(A + st->off[SC_S]);
    float* conv = reinterpret_cast<float*>(A + st->off[SC_CONV]);
    bf16_t* kv = reinterpret_cast<bf16_t*>(A + st->off[SC_KV]);
    int32_t* pos = reinterpret_cast<int32_t*>(A + st->off[SC_POS]);
    bf16_t* resid = reinterpret_cast<bf16_t*>(A + st->off[SC_RESID]);
    float* proj = reinterpret_cast<float*>(A + st->off[SC_PROJ]);
    float* obuf = reinterpret_cast<float*>(A + st->off[SC_O]);
    float* qrot = reinterpret_cast<float*>(A + st->off[SC_QROT]);
    bf16_t* attn = reinterpret_cast<bf16_t*>(A + st->off[SC_ATTN]);
    float* part = reinterpret_cast<float*>(A + st->off[SC_PART]);
    bf16_t* mlp = reinterpret_cast<bf16_t*>(A + st->off[SC_MLP]);
    float* bestv = reinterpret_cast<float*>(A + st->off[SC_BESTV]);
    int32_t* besti = reinterpret_cast<int32_t*>(A + st->off[SC_BESTI]);
    void* ws = A + st->off[SC_WS];
    const size_t ws_bytes = st->off[SC_BAR] - st->off[SC_WS];
    bf16_t* gn_rows = reinterpret_cast<bf16_t*>(A + st->off[SC_GN]);
    bf16_t* xn_rows = reinterpret_cast<bf16_t*>(A + st->off[SC_XN]);
    const int64_t proj_ld = std::max(d.gdn_out, d.attn_out);
    const float eps = m->cfg.norm_eps;
    const bool many = M > SK_MAXM;  // norms once per row, then plain-input GEMVs
    auto norm_rows = [&](const bf16_t* gains, bool embed) -> int {
        NormRowsParams q{resid, d.D, tokens, m->embed, d.V, resid, d.D, gains, eps, xn_rows, d.D, M, d.D, status_dev};
        cudaError_t e = embed ? launch_pdl(k_norm_rows<true>, dim3((M + 7) / 8), dim3(256), 0, s, q)
                              : launch_pdl(k_norm_rows<false>, dim3((M + 7) / 8), dim3(256), 0, s, q);
        return launch_status(e);
    };
    const size_t s_layer = (size_t)B * d.H * d.dv * d.dk;
    const size_t c_layer = (size_t)B * (d.kc - 1) * d.C;
    const size_t kv_half = (size_t)B * d.nkv * Lmax * d.hd;
    const size_t srec_layer = (size_t)B * T * d.H * d.dv * d.dk;
    const size_t trec_layer = (size_t)B * T * (d.kc - 1) * d.C;
    const VerifyLayout vlay = verify_layout(d, B, T);
    int ig = 0, ia = 0;
    for (int l = 0; l < layer_begin; ++l) (is_attn_layer(&m->cfg, l) ? ia : ig)++;
    for (int l = layer_begin; l < layer_end; ++l) {
        const uint16_t* const* w = m->w[l];
        const bool att = is_attn_layer(&m->cfg, l);
        // input RMSNorm + in-projection (layer 0 gathers the embedding rows); in a
        // GDN layer the epilogue also runs the causal conv of the q|k|v channels
        {
            GemvParams p = {};
            p.W = w[HGD_W_IN]; p.packed = 1; p.N = (int)(att ? d.attn_out : d.gdn_out); p.K = d.D;
            p.x = resid; p.x_ld = d.D; p.norm_w = w[HGD_W_IN_NORM]; p.eps = eps;
            p.y = proj; p.y_ld = proj_ld; p.status = status_dev;
            if (att) {
                p.rope_nq = d.nq; p.rope_nkv = d.nkv; p.rope_hd = d.hd; p.rope_Lmax = Lmax;
                p.rope_inv1 = rope_inv1_of(d, m->cfg.rope_base); p.rope_q = qrot;
                p.rope_k = kv + (size_t)ia * 2 * kv_half; p.rope_v = p.rope_k + kv_half;
                p.rope_pos = pos; p.conv_T = T;
            }
            if (l == 0) {
                p.tokens = tokens; p.embed = m->embed; p.vocab = d.V; p.resid_out = resid; p.resid_out_ld = d.D;
            }
            if (many) {
                if ((rc = norm_rows(w[HGD_W_IN_NORM], l == 0))) return rc;
                p.x = xn_rows;
            }
            if (!att) {
                p.conv_w = w[HGD_W_CONV]; p.conv_tail = conv + ig * c_layer;
                p.conv_rec = tail_rec ? tail_rec + ig * trec_layer : nullptr;
                if (vl) {
                    p.conv_tail = reinterpret_cast<float*>(vl + vlay.conv) + ig * c_layer;
                    p.conv_xlog = reinterpret_cast<float*>(vl + vlay.layer(ig) + vlay.x);
                }
                p.conv_C = (int)d.C; p.conv_T = T;
                rc = many     ? run_gemv<PRO_COPY, EPI_QKV_CONV>(p, M, di.sms, ws, ws_bytes, s)
                     : (l == 0) ? run_gemv<PRO_EMBED_RMSNORM, EPI_QKV_CONV>(p, M, di.sms, ws, ws_bytes, s)
                                : run_gemv<PRO_RMSNORM, EPI_QKV_CONV>(p, M, di.sms, ws, ws_bytes, s);
            } else {
                rc = many     ? run_gemv<PRO_COPY, EPI_ROPE>(p, M, di.sms, ws, ws_bytes, s)
                     : (l == 0) ? run_gemv<PRO_EMBED_RMSNORM, EPI_ROPE>(p, M, di.sms, ws, ws_bytes, s)
                                : run_gemv<PRO_RMSNORM, EPI_ROPE>(p, M, di.sms, ws, ws_bytes, s);
            }
            if (rc) return rc;
        }
        if (!att) {
            GdnLayerParams g{};
            g.proj = proj; g.proj_ld = proj_ld;
            g.A_log = w[HGD_W_A_LOG]; g.dt_bias = w[HGD_W_DT_BIAS];
            g.S = Sall + ig * s_layer;
            g.o = obuf; g.o_ld = (int64_t)d.H * d.dv;
            g.S_rec = S_rec ? S_rec + ig * srec_layer : nullptr;
            g.B = B; g.T = T; g.H = d.H; g.dv = d.dv; g.Hk = d.Hk;
            if (vl) {
                g.log_alpha = reinterpret_cast<float*>(vl + vlay.layer(ig) + vlay.alpha);
                g.log_delta = reinterpret_cast<float*>(vl + vlay.layer(ig) + vlay.delta);
                g.log_k = reinterpret_cast<float*>(vl + vlay.layer(ig) + vlay.k);
            }
            if ((rc = launch_status(launch_gdn_layer(d, B, g, s)))) return rc;
            GemvParams p = {};
            p.W = w[HGD_W_OUT]; p.packed = 1; p.N = d.D; p.K = d.H * d.dv;
            p.y = resid; p.y_ld = d.D; p.resid = resid; p.resid_ld = d.D; p.status = status_dev;
            if (M > SK_MAXM) {
                // many rows: the gated norm once per (row, head), then a plain-input GEMV
                // (the same values reach the MMAs as from the fused prologue)
                GatedNormParams g{obuf, (int64_t)d.H * d.dv, proj + d.C, proj_ld, w[HGD_W_GNORM], gn_rows,
                                  (int64_t)d.H * d.dv, M, d.H, d.dv, eps};
                cudaError_t e = launch_pdl(k_gated_norm, dim3((M * d.H + 7) / 8), dim3(256), 0, s, g);
                if (e != cudaSuccess) return launch_status(e);
                p.x = gn_rows; p.x_ld = (int64_t)d.H * d.dv;
                if ((rc = run_gemv<PRO_COPY, EPI_RESID>(p, M, di.sms, ws, ws_bytes, s))) return rc;
            } else {
                p.o = obuf; p.o_ld = (int64_t)d.H * d.dv;
                p.z = proj + d.C; p.z_ld = proj_ld; p.gnorm_w = w[HGD_W_GNORM]; p.gn_d = d.dv; p.eps = eps;
                if ((rc = run_gemv<PRO_GATED_NORM, EPI_RESID>(p, M, di.sms, ws, ws_bytes, s))) return rc;
            }
            ++ig;
        } else {
            AttnParams a{};
            a.proj = proj; a.proj_ld = proj_ld; a.qrot = qrot;
            a.kcache = kv + (size_t)ia * 2 * kv_half; a.vcache = a.kcache + kv_half;
            a.pos = pos; a.part = part; a.out = attn; a.status = status_dev;
            a.B = B; a.T = T; a.nq = d.nq; a.nkv = d.nkv; a.hd = d.hd; a.Lmax = Lmax;
            a.max_chunks = max_chunks_of(Lmax);
            cudaError_t e = launch_pdl(k_attn_partial, dim3(B, d.nkv, a.max_chunks), dim3(32 * ATTN_PART_WARPS),
                                       attn_part_smem_bytes(d.hd), s, a);
            if ((rc = launch_status(e))) return rc;
            e = launch_pdl(k_attn_merge, dim3(M, d.nq), dim3(d.hd), 0, s, a);
            if ((rc = launch_status(e))) return rc;
            GemvParams p = {};
            p.W = w[HGD_W_OUT]; p.packed = 1; p.N = d.D; p.K = d.nq * d.hd;
            p.x = attn; p.x_ld = (int64_t)d.nq * d.hd;
            p.y = resid; p.y_ld = d.D; p.resid = resid; p.resid_ld = d.D; p.status = status_dev;
            if ((rc = run_gemv<PRO_COPY, EPI_RESID>(p, M, di.sms, ws, ws_bytes, s))) return rc;
            ++ia;
        }
        // MLP: RMSNorm + fused up/gate SwiGLU, then down + residual
        {
            GemvParams p = {};
            p.W = w[HGD_W_GATE]; p.packed = 1; p.N = d.I; p.K = d.D;
            p.x = resid; p.x_ld = d.D; p.norm_w = w[HGD_W_POST_NORM]; p.eps = eps;
            p.y = mlp; p.y_ld = d.I; p.status = status_dev;
            if (many) {
                if ((rc = norm_rows(w[HGD_W_POST_NORM], false))) return rc;
                p.x = xn_rows;
                if ((rc = run_gemv<PRO_COPY, EPI_SWIGLU>(p, M, di.sms, ws, ws_bytes, s))) return rc;
            } else if ((rc = run_gemv<PRO_RMSNORM, EPI_SWIGLU>(p, M, di.sms, ws, ws_bytes, s))) {
                return rc;
            }
        }
        {
            GemvParams p = {};
            p.W = w[HGD_W_DOWN]; p.packed = 1; p.N = d.D; p.K = d.I;
            p.x = mlp; p.x_ld = d.I;
            p.y = resid; p.y_ld = d.D; p.resid = resid; p.resid_ld = d.D; p.status = status_dev;
            if ((rc = run_gemv<PRO_COPY, EPI_RESID>(p, M, di.sms, ws, ws_bytes, s))) return rc;
        }
    }
    // final norm + tied LM head + per-CTA argmax, then the row argmax
    if (run_head) {
        GemvParams p = {};
        p.W = m->lm_head ? m->lm_head : m->embed; p.packed = 1; p.N = d.V; p.K = d.D;
        p.x = resid; p.x_ld = d.D; p.norm_w = m->final_norm; p.eps = eps;
        p.logits = logits; p.logits_ld = d.V; p.best_v = bestv; p.best_i = besti; p.status = status_dev;
        int G = 0;
        if (many) {
            if ((rc = norm_rows(m->final_norm, false))) return rc;
            p.x = xn_rows;
            if ((rc = run_gemv<PRO_COPY, EPI_ARGMAX>(p, M, di.sms, nullptr, 0, s, &G))) return rc;
        } else if ((rc = run_gemv<PRO_RMSNORM, EPI_ARGMAX>(p, M, di.sms, nullptr, 0, s, &G))) {
            return rc;
        }
        cudaError_t e = launch_pdl(k_argmax_finalize, dim3(M), dim3(128), 0, s, (const float*)bestv,
                                   (const int32_t*)besti, G, M, argmax, status_dev, vl ? nullptr : pos, B, T);
        if ((rc = launch_status(e))) return rc;
    }
    return HGD_OK;
}

int hgd_decode_layer_stack_range(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T,
                                 int layer_begin, int layer_end, int run_head, float* logits, int32_t* argmax,
                                 float* S_rec, float* tail_rec, int32_t* status_dev, hgd_stream_t stream) {
    return chain_run(m, st, tokens, T, layer_begin, layer_end, run_head, logits, argmax, S_rec, tail_rec, status_dev,
                     stream, nullptr);
}

int hgd_verify_log_bytes(const hgd_config* cfg, int B, int T, size_t* bytes) {
    if (!bytes) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if (B < 1 || T < 1) return HGD_ERR_INVALID_ARG;
    if ((int64_t)B * T > 256) return HGD_ERR_UNSUPPORTED_SHAPE;
    *bytes = verify_layout(d, B, T).total;
    return HGD_OK;
}

int hgd_decode_layer_stack_verify(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T,
                                  float* logits, int32_t* argmax, void* log, size_t log_bytes, int32_t* status_dev,
                                  hgd_stream_t stream) {
    if (!m || !st || !st->arena || !tokens || !argmax || !log) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (reinterpret_cast<uintptr_t>(log) & 255u) return HGD_ERR_MISALIGNED;
    const VerifyLayout vlay = verify_layout(d, st->B, T);
    if (log_bytes < vlay.total) return HGD_ERR_BUFFER_TOO_SMALL;
    uint8_t* vl = static_cast<uint8_t*>(log);
    const uint8_t* A = static_cast<const uint8_t*>(st->arena);
    // the window's conv runs on a copy of the tails; the state's own stay as they are
    if (d.n_gdn > 0 && cudaMemcpyAsync(vl + vlay.conv, A + st->off[SC_CONV],
                                       (size_t)d.n_gdn * st->B * (d.kc - 1) * d.C * 4, cudaMemcpyDeviceToDevice,
                                       (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    return chain_run(m, st, tokens, T, 0, d.L, 1, logits, argmax, nullptr, nullptr, status_dev, stream, vl);
}

int hgd_decode_layer_stack_keep(const hgd_model* m, const hgd_state* st, int T, const void* log, size_t log_bytes,
                                const int32_t* keep, int32_t* status_dev, hgd_stream_t stream) {
    if (!m || !st || !st->arena || !log || !keep) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if ((reinterpret_cast<uintptr_t>(log) & 255u) || !al16(keep) || (status_dev && !al16(status_dev)))
        return HGD_ERR_MISALIGNED;
    const int B = st->B;
    const VerifyLayout vlay = verify_layout(d, B, T);
    if (log_bytes < vlay.total) return HGD_ERR_BUFFER_TOO_SMALL;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    const uint8_t* vl = static_cast<const uint8_t*>(log);
    uint8_t* A = static_cast<uint8_t*>(st->arena);
    float* Sall = reinterpret_cast<float*>(A + st->off[SC_S]);
    float* conv = reinterpret_cast<float*>(A + st->off[SC_CONV]);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t s_layer = (size_t)B * d.H * d.dv * d.dk;
    const size_t c_layer = (size_t)B * (d.kc - 1) * d.C;
    for (int ig = 0; ig < d.n_gdn; ++ig) {
        const uint8_t* ly = vl + vlay.layer(ig);
        GdnKeepParams g{Sall + ig * s_layer, reinterpret_cast<const float*>(ly + vlay.alpha),
                        reinterpret_cast<const float*>(ly + vlay.delta), reinterpret_cast<const float*>(ly + vlay.k),
                        keep, status_dev, B, T, d.H, d.dv};
        const dim3 grid(B * d.H, d.dv / GDN_ROWS), block(GDN_WARPS * 32);
        cudaError_t e;
        switch (d.dk) {
            case 32: e = launch_pdl(k_gdn_keep<1>, grid, block, 0, s, g); break;
            case 64: e = launch_pdl(k_gdn_keep<2>, grid, block, 0, s, g); break;
            case 128: e = launch_pdl(k_gdn_keep<4>, grid, block, 0, s, g); break;
            default: e = launch_pdl(k_gdn_keep<8>, grid, block, 0, s, g); break;
        }
        if ((rc = launch_status(e))) return rc;
        ConvKeepParams c{conv + ig * c_layer, reinterpret_cast<const float*>(ly + vlay.x), keep, status_dev,
                         B, T, (int)d.C, d.kc};
        const int64_t n = (int64_t)B * d.C;
        e = launch_pdl(k_conv_keep, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, c);
        if ((rc = launch_status(e))) return rc;
    }
    int32_t* pos = reinterpret_cast<int32_t*>(A + st->off[SC_POS]);
    return launch_status(launch_pdl(k_pos_keep, dim3(1), dim3(32), 0, s, pos, keep, status_dev, B, T));
}

// ------------------------------------------------- tensor-core decode chain

int hgd_model_tc_bytes(const hgd_config* cfg, size_t* bytes) {
    if (!bytes) return HGD_ERR_INVALID_ARG;
    Dims d;
    int rc = dims_of(cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    if (d.D % TC_BK || d.I % TC_BK || (d.H * d.dv) % TC_BK || (d.nq * d.hd) % TC_BK) return HGD_ERR_UNSUPPORTED_SHAPE;
    *bytes = tc_walk(d, cfg, -2, -2, nullptr);
    return HGD_OK;
}

int hgd_model_tc_load(const hgd_config* cfg, void* tc_arena, size_t bytes, int layer, int tensor,
                      const uint16_t* src, hgd_stream_t stream) {
    size_t need = 0;
    int rc = hgd_model_tc_bytes(cfg, &need);
    if (rc) return rc;
    if (!tc_arena || !src) return HGD_ERR_INVALID_ARG;
    if (bytes < need) return HGD_ERR_BUFFER_TOO_SMALL;
    if ((reinterpret_cast<uintptr_t>(tc_arena) & 255u) || !al16(src)) return HGD_ERR_MISALIGNED;
    Dims d;
    dims_of(cfg, &d);
    if (layer < -1 || layer >= d.L) return HGD_ERR_INVALID_ARG;
    int which = -1;
    int64_t N = 0, K = 0;
    int half = -1;
    if (layer == -1) {
        if (tensor != (d.untied ? HGD_W_LM_HEAD : HGD_W_EMBED)) return HGD_ERR_INVALID_ARG;
        N = d.V; K = d.D;
    } else {
        const bool att = is_attn_layer(cfg, layer);
        switch (tensor) {
            case HGD_W_IN: which = 0; N = att ? d.attn_out : d.gdn_out; K = d.D; break;
            case HGD_W_OUT: which = 1; N = d.D; K = att ? (int64_t)d.nq * d.hd : (int64_t)d.H * d.dv; break;
            case HGD_W_GATE: which = 2; N = d.I; K = d.D; half = 0; break;
            case HGD_W_UP: which = 2; N = d.I; K = d.D; half = 1; break;
            case HGD_W_DOWN: which = 3; N = d.D; K = d.I; break;
            default: return HGD_ERR_INVALID_ARG;
        }
    }
    size_t off = 0;
    tc_walk(d, cfg, layer, which, &off);
    uint16_t* dst = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(tc_arena) + off);
    if (half < 0) return hgd_gemm_tc_pack_weight(src, dst, (int)N, (int)K, stream);
    const int64_t chunks = tc_rows64(N) * (K / 8);
    k_tc_pack_w_swiglu<<<(unsigned)std::min<int64_t>(4736, (chunks + 255) / 256), 256, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<const bf16_t*>(src), reinterpret_cast<bf16_t*>(dst), (int)N, (int)K, half);
    return launch_status(cudaGetLastError());
}

int hgd_model_attach_tc(hgd_model* m, const void* tc_arena, size_t bytes) {
    if (!m || !tc_arena) return HGD_ERR_INVALID_ARG;
    size_t need = 0;
    int rc = hgd_model_tc_bytes(&m->cfg, &need);
    if (rc) return rc;
    if (bytes < need) return HGD_ERR_BUFFER_TOO_SMALL;
    if (reinterpret_cast<uintptr_t>(tc_arena) & 255u) return HGD_ERR_MISALIGNED;
    Dims d;
    dims_of(&m->cfg, &d);
    const uint8_t* base = static_cast<const uint8_t*>(tc_arena);
    size_t off = 0;
    tc_walk(d, &m->cfg, -1, 0, &off);
    m->tc_head = reinterpret_cast<const uint16_t*>(base + off);
    for (int l = 0; l < d.L; ++l)
        for (int w = 0; w < 4; ++w) {
            tc_walk(d, &m->cfg, l, w, &off);
            m->tcw[l][w] = reinterpret_cast<const uint16_t*>(base + off);
        }
    return HGD_OK;
}

int hgd_decode_layer_stack_tc(const hgd_model* m, const hgd_state* st, const int32_t* tokens, int T, float* logits,
                              int32_t* argmax, float* S_rec, float* tail_rec, int32_t* status_dev,
                              hgd_stream_t stream) {
    if (!m || !st || !st->arena || !tokens || !argmax) return HGD_ERR_INVALID_ARG;
    if (T < 1 || T > st->Tmax) return HGD_ERR_INVALID_ARG;
    if (!m->tc_head) return HGD_ERR_INVALID_ARG;  // no tensor-core weights attached
    Dims d;
    int rc = dims_of(&m->cfg, &d);
    if (rc) return rc;
    if ((rc = check_supported(d))) return rc;
    const int B = st->B, M = B * T, Lmax = st->Lmax;
    if (M > TC_MAXN) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(tokens) || !al16(argmax) || (logits && !al16(logits)) || (S_rec && !al16(S_rec)) ||
        (tail_rec && !al16(tail_rec)))
        return HGD_ERR_MISALIGNED;
    DevInfo di;
    if ((rc = device_info(&di))) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* A = static_cast<uint8_t*>(st->arena);
    float* Sall = reinterpret_cast<float*>(A + st->off[SC_S]);
    float* conv = reinterpret_cast<float*>(A + st->off[SC_CONV]);
    bf16_t* kv = reinterpret_cast<bf16_t*>(A + st->off[SC_KV]);
    int32_t* pos = reinterpret_cast<int32_t*>(A + st->off[SC_POS]);
    bf16_t* resid = reinterpret_cast<bf16_t*>(A + st->off[SC_RESID]);
    float* proj = reinterpret_cast<float*>(A + st->off[SC_PROJ]);
    float* obuf = reinterpret_cast<float*>(A + st->off[SC_O]);
    float* qrot = reinterpret_cast<float*>(A + st->off[SC_QROT]);
    bf16_t* attn = reinterpret_cast<bf16_t*>(A + st->off[SC_ATTN]);
    float* part = reinterpret_cast<float*>(A + st->off[SC_PART]);
    bf16_t* mlp = reinterpret_cast<bf16_t*>(A + st->off[SC_MLP]);
    bf16_t* gn_rows = reinterpret_cast<bf16_t*>(A + st->off[SC_GN]);
    bf16_t* xn_rows = reinterpret_cast<bf16_t*>(A + st->off[SC_XN]);
    float* ty = reinterpret_cast<float*>(A + st->off[SC_TCY]);
    float* lg = logits ? logits : reinterpret_cast<float*>(A + st->off[SC_TCLOG]);
    const float eps = m->cfg.norm_eps;
    const int64_t Ih = tc_rows64(d.I);
    // every GEMM input is written straight into the GEMM's packed layout (NTp
    // rows; the rows past M are never read back into a result)
    const int NTp = tc_ntp(M);
    auto norm_rows = [&](const bf16_t* gains, bool embed) -> int {
        NormRowsParams q{resid, d.D, tokens, m->embed, d.V, resid, d.D, gains, eps, xn_rows, d.D, M, d.D, status_dev,
                         NTp};
        cudaError_t e = embed ? launch_pdl(k_norm_rows<true>, dim3((M + 7) / 8), dim3(256), 0, s, q)
                              : launch_pdl(k_norm_rows<false>, dim3((M + 7) / 8), dim3(256), 0, s, q);
        return launch_status(e);
    };
    auto gemm = [&](const uint16_t* Wp, const bf16_t* x, int64_t x_ld, float* y, int N, int K) -> int {
        return tc_run(reinterpret_cast<const bf16_t*>(Wp), x, x_ld, y, M, N, K, nullptr, status_dev, s, nullptr, true);
    };
    // a projection added to the residual rows (ty is its scratch)
    auto gemm_resid = [&](const uint16_t* Wp, const bf16_t* x, int64_t x_ld, int K) -> int {
        return tc_run(reinterpret_cast<const bf16_t*>(Wp), x, x_ld, ty, M, d.D, K, nullptr, status_dev, s, resid, true);
    };
    const size_t s_layer = (size_t)B * d.H * d.dv * d.dk;
    const size_t c_layer = (size_t)B * (d.kc - 1) * d.C;
    const size_t kv_half = (size_t)B * d.nkv * Lmax * d.hd;
    const size_t srec_layer = (size_t)B * T * d.H * d.dv * d.dk;
    const size_t trec_layer = (size_t)B * T * (d.kc - 1) * d.C;
    int ig = 0, ia = 0;
    for (int l = 0; l < d.L; ++l) {
        const uint16_t* const* w = m->w[l];
        const bool att = is_attn_layer(&m->cfg, l);
        const int Nin = (int)(att ? d.attn_out : d.gdn_out);
        // RMSNorm once per row (layer 0 gathers the embedding rows), the in-projection
        if ((rc = norm_rows(w[HGD_W_IN_NORM], l == 0))) return rc;
        if ((rc = gemm(m->tcw[l][0], xn_rows, d.D, proj, Nin, d.D))) return rc;
        if (!att) {
            // the conv runs inside the GDN kernel where one CTA holds a head's q, k and
            // v channels alone (dk = dv = 128, a key head per value head)
            const bool fused_conv = d.dv == GDN_FUSED_DV && d.dk == 128 && d.Hk == d.H;
            if (!fused_conv) {
                TcConvParams cp{proj, Nin, conv + ig * c_layer, w[HGD_W_CONV],
                                tail_rec ? tail_rec + ig * trec_layer : nullptr, B, T, (int)d.C};
                const int64_t n = (int64_t)B * d.C;
                const dim3 cg((unsigned)((n + 255) / 256)), cb(256);
                if ((rc = launch_status(tail_rec ? launch_pdl(k_tc_conv<true>, cg, cb, 0, s, cp)
                                                 : launch_pdl(k_tc_conv<false>, cg, cb, 0, s, cp))))
                    return rc;
            }
            GdnLayerParams g{};
            g.proj = proj; g.proj_ld = Nin;
            g.A_log = w[HGD_W_A_LOG]; g.dt_bias = w[HGD_W_DT_BIAS];
            g.S = Sall + ig * s_layer;
            g.o = obuf; g.o_ld = (int64_t)d.H * d.dv;
            g.S_rec = S_rec ? S_rec + ig * srec_layer : nullptr;
            g.B = B; g.T = T; g.H = d.H; g.dv = d.dv; g.Hk = d.Hk;
            if (d.dv == GDN_FUSED_DV && d.dk <= 128) {
                // one CTA per (stream, head) forms the gated norm too, packed for the GEMM
                g.z = proj + d.C; g.z_ld = Nin; g.gn_w = w[HGD_W_GNORM]; g.u = gn_rows; g.u_ntp = NTp; g.eps = eps;
                const dim3 grid(B * d.H), block(GDN_FUSED_DV / 8 * 32);
                cudaError_t e;
                if (fused_conv) {
                    g.conv_tail = conv + ig * c_layer; g.conv_w = w[HGD_W_CONV];
                    g.conv_tail_rec = tail_rec ? tail_rec + ig * trec_layer : nullptr; g.C = (int)d.C;
                    e = launch_pdl(k_gdn_layer<4, 8, GDN_FUSED_DV / 8, true, true>, grid, block, 0, s, g);
                } else switch (d.dk) {
                    case 32: e = launch_pdl(k_gdn_layer<1, 8, GDN_FUSED_DV / 8, true>, grid, block, 0, s, g); break;
                    case 64: e = launch_pdl(k_gdn_layer<2, 8, GDN_FUSED_DV / 8, true>, grid, block, 0, s, g); break;
                    default: e = launch_pdl(k_gdn_layer<4, 8, GDN_FUSED_DV / 8, true>, grid, block, 0, s, g); break;
                }
                if ((rc = launch_status(e))) return rc;
            } else {
                if ((rc = launch_status(launch_gdn_layer(d, B, g, s)))) return rc;
                GatedNormParams gq{obuf, (int64_t)d.H * d.dv, proj + d.C, Nin, w[HGD_W_GNORM], gn_rows,
                                   (int64_t)d.H * d.dv, M, d.H, d.dv, eps, NTp};
                cudaError_t e = launch_pdl(k_gated_norm, dim3((M * d.H + 7) / 8), dim3(256), 0, s, gq);
                if ((rc = launch_status(e))) return rc;
            }
            if ((rc = gemm_resid(m->tcw[l][1], gn_rows, (int64_t)d.H * d.dv, d.H * d.dv))) return rc;
            ++ig;
        } else {
            TcRopeParams rp{proj, Nin, qrot, kv + (size_t)ia * 2 * kv_half, kv + (size_t)ia * 2 * kv_half + kv_half,
                            pos, status_dev, T, d.nq, d.nkv, d.hd, Lmax, rope_inv1_of(d, m->cfg.rope_base)};
            if ((rc = launch_status(launch_pdl(k_tc_rope, dim3(M), dim3(256), 0, s, rp)))) return rc;
            AttnParams a{};
            a.proj = proj; a.proj_ld = Nin; a.qrot = qrot;
            a.kcache = kv + (size_t)ia * 2 * kv_half; a.vcache = a.kcache + kv_half;
            a.pos = pos; a.part = part; a.out = attn; a.status = status_dev;
            a.B = B; a.T = T; a.nq = d.nq; a.nkv = d.nkv; a.hd = d.hd; a.Lmax = Lmax;
            a.max_chunks = max_chunks_of(Lmax);
            a.pack_ntp = NTp;
            if ((rc = launch_status(launch_attn_partial_tc(d.hd, dim3(B, d.nkv, a.max_chunks), s, a)))) return rc;
            cudaError_t e = launch_pdl(k_attn_merge, dim3(M, d.nq), dim3(d.hd), 0, s, a);
            if ((rc = launch_status(e))) return rc;
            if ((rc = gemm_resid(m->tcw[l][1], attn, (int64_t)d.nq * d.hd, d.nq * d.hd))) return rc;
            ++ia;
        }
        // MLP: RMSNorm once per row, gate and up in one GEMM whose epilogue forms the
        // SwiGLU rows (packed for the down GEMM), down + residual
        if ((rc = norm_rows(w[HGD_W_POST_NORM], false))) return rc;
        if ((rc = tc_run(reinterpret_cast<const bf16_t*>(m->tcw[l][2]), xn_rows, d.D, nullptr, M, (int)(2 * Ih),
                         d.D, nullptr, status_dev, s, nullptr, true, mlp, d.I)))
            return rc;
        if ((rc = gemm_resid(m->tcw[l][3], mlp, d.I, d.I))) return rc;
    }
    // final RMSNorm, the head, the argmax of each row, the positions
    if ((rc = norm_rows(m->final_norm, false))) return rc;
    if ((rc = gemm(m->tc_head, xn_rows, d.D, lg, d.V, d.D))) return rc;
    // the argmax partials in the projection scratch (free after the last layer)
    float* am_v = ty;
    int* am_i = reinterpret_cast<int*>(ty + (size_t)M * TC_AM_SLICES);
    if ((rc = launch_status(launch_pdl(k_tc_argmax_part, dim3(M, TC_AM_SLICES), dim3(256), 0, s, (const float*)lg,
                                       (int64_t)d.V, d.V, am_v, am_i))))
        return rc;
    return launch_status(launch_pdl(k_tc_argmax_final, dim3(M), dim3(32), 0, s, (const float*)am_v, (const int*)am_i,
                                    argmax, status_dev, pos, B, T));
}

}  // extern "C"

// ====================================================== allocation-free GEMV
// Some callers cannot allocate device memory at all: a plugin hosted by a
// framework that owns the device allocator and gives the plugin no handle to
// it, or a latency-critical decode loop in which a cudaMalloc would synchronise
// the device and stall every stream.  For them hgd_gemv_bf16_static_ws runs the
// GEMV with its split-K scratch in a fixed array that is part of the library
// image: nothing is allocated per call, and the caller passes only its inputs
// and its output.  The array (kStaticWsBytes) lives on every device that loads
// the library until the process exits, and every call shares it.

namespace {

constexpr size_t kStaticWsBytes = (size_t)4 << 20;  // 4 MiB of scratch per device
static __device__ __align__(256) uint8_t g_gemv_static_ws[kStaticWsBytes];

// Device address of the array in the current context, looked up once per
// context with that context current (host code cannot use the symbol itself: it
// names a host-side stand-in).  Keyed on the context, not the device: after a
// device reset the array is loaded again, possibly elsewhere, and the next call
// looks it up afresh.  The cache is guarded by a mutex, so first calls from
// several host threads are safe.
int static_ws_address(void** out) {
    static CtxCache<void*> addr;
    void* p = nullptr;
    if (addr.get(current_ctx_id(), &p) && p) { *out = p; return HGD_OK; }
    if (cudaGetSymbolAddress(&p, g_gemv_static_ws) != cudaSuccess || !p) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    addr.put(current_ctx_id(), p);  // the lookup has made the context current if it was not
    *out = p;
    return HGD_OK;
}

}  // namespace

extern "C" int hgd_gemv_bf16_static_ws(const uint16_t* W, const uint16_t* x, void* y, int y_is_fp32, int M,
                                       int N, int K, hgd_stream_t stream) {
    if (!W || !x || !y || M < 1 || N < 1 || K < 1) return HGD_ERR_INVALID_ARG;
    if (K % 32 != 0 || K > 65536) return HGD_ERR_UNSUPPORTED_SHAPE;
    if (!al16(W) || !al16(x) || !al16(y)) return HGD_ERR_MISALIGNED;
    DevInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    const size_t need = gemv_ws_bytes(M, N, K, false);
    if (need > kStaticWsBytes) return HGD_ERR_BUFFER_TOO_SMALL;
    void* ws = nullptr;
    if ((rc = static_ws_address(&ws))) return rc;
    // the row-block counters must start at zero; the partials need no clearing
    if (need && cudaMemsetAsync(ws, 0, kWsCounterBytes, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return HGD_ERR_CUDA;
    }
    GemvParams p = {};
    p.W = W; p.N = N; p.K = K; p.x = x; p.x_ld = K; p.y = y; p.y_ld = N;
    if (y_is_fp32)
        return run_gemv<PRO_COPY, EPI_F32>(p, M, di.sms, need ? ws : nullptr, need, (cudaStream_t)stream);
    return run_gemv<PRO_COPY, EPI_BF16>(p, M, di.sms, need ? ws : nullptr, need, (cudaStream_t)stream);
}
