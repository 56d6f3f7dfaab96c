// zha_abi.cu -- the C ABI (include/zha.h): argument checks, buffer layouts and
// kernel launches.  Every step of the path runs in the kernels included below;
// this file only validates, lays out the caller's buffers and launches.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "zha.h"
#include "zha_common.cuh"
#include "zha_build.cuh"
#include "zha_plan.cuh"
#include "zha_route.cuh"
#include "zha_attend.cuh"
#include "zha_attend_tc.cuh"
#include "zha_prefill.cuh"
#include "zha_score_tc.cuh"

using namespace zha;

namespace {

thread_local char g_err[512] = "";

// An NVTX range around one C-ABI call, so that a profiler's timeline names the call
// each kernel belongs to (free when no tool is attached).
struct Range {
    explicit Range(const char* name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range&) = delete;
    Range& operator=(const Range&) = delete;
};

// Bound of the tensor-core decode attention's waits on another warp's progress
// (zha_set_wait_limit); waits on the kernel's own copies and MMAs keep kWaitLongNs.
std::atomic<uint64_t> g_wait_ns{kWaitLongNs};

int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

#define ZHA_CUDA(call)                                                                   \
    do {                                                                                 \
        cudaError_t e_ = (call);                                                         \
        if (e_ != cudaSuccess) return fail(ZHA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

#define ZHA_TRY(expr)               \
    do {                            \
        int r_ = (expr);            \
        if (r_ != ZHA_OK) return r_; \
    } while (0)

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct TreeLayout {
    int Lcap, R, vsum;
    int64_t ncap[kMaxLevels];
    size_t off_ntree, off_qref, off_khat[kMaxLevels], off_bhat[kMaxLevels], off_vhat[kMaxLevels], total;
};

struct WsLayout {
    int64_t cand_cap, par_cap, kb_cap, sel_cap, item_cap, words;
    size_t off_scores, off_parents, off_sel, off_count, off_items, off_nitems, off_ml, off_acc, off_counters;
    size_t off_rows, off_cand, off_ballot, off_scanned, off_pr_ml, off_pr_acc;
    size_t total;
};


int validate(const zha_config* c) {
    if (!c) return fail(ZHA_ERR_INVALID_ARG, "cfg is null");
    if (c->d != 64 && c->d != 128) return fail(ZHA_ERR_UNSUPPORTED, "d=%d: head dim must be 64 or 128", c->d);
    if (c->Hq < 1 || c->Hkv < 1 || c->Hq % c->Hkv) return fail(ZHA_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d", c->Hq, c->Hkv);
    const int G = c->Hq / c->Hkv;
    if (G != 1 && G != 2 && G != 4) return fail(ZHA_ERR_UNSUPPORTED, "Hq/Hkv=%d: groups of 1, 2 or 4 query heads", G);
    if (c->Hkv > 32) return fail(ZHA_ERR_UNSUPPORTED, "Hkv=%d > 32", c->Hkv);
    if (c->B < 1) return fail(ZHA_ERR_INVALID_ARG, "B=%d", c->B);
    if (c->B > 256) return fail(ZHA_ERR_UNSUPPORTED, "B=%d > 256", c->B);
    if (c->b < 2 || c->b > 32) return fail(c->b < 2 ? ZHA_ERR_INVALID_ARG : ZHA_ERR_UNSUPPORTED, "b=%d: branching must be 2..32", c->b);
    if (c->R < 1) return fail(ZHA_ERR_INVALID_ARG, "R=%d", c->R);
    if (c->R > 16) return fail(ZHA_ERR_UNSUPPORTED, "R=%d: at most 16 reference queries per node", c->R);
    if (c->dtype != ZHA_F32 && c->dtype != ZHA_BF16) return fail(ZHA_ERR_INVALID_ARG, "dtype=%d", c->dtype);
    if (c->batch < 1) return fail(ZHA_ERR_INVALID_ARG, "batch=%d", c->batch);
    if (c->N_cap < 1 || c->N_cap > (int64_t{1} << 31) - 128) return fail(ZHA_ERR_INVALID_ARG, "N_cap=%lld", (long long)c->N_cap);
    if (c->L_fixed < 0 || c->L_fixed > ZHA_MAX_LEVELS) return fail(ZHA_ERR_INVALID_ARG, "L_fixed=%d", c->L_fixed);
    if (c->vsum != 0 && c->vsum != 1) return fail(ZHA_ERR_INVALID_ARG, "vsum=%d must be 0 or 1", c->vsum);
    if (c->vsum && c->R != 1) return fail(ZHA_ERR_UNSUPPORTED, "vsum=1: value summaries take R = 1 (R=%d)", c->R);
    if (!(c->scale >= 0.f) || !std::isfinite(c->scale)) return fail(ZHA_ERR_INVALID_ARG, "scale must be finite and >= 0");
    int64_t n[kMaxLevels];
    const int L = tree_levels(c->N_cap, c->B, c->b, c->L_fixed, n);
    if (L < 0) return fail(ZHA_ERR_UNSUPPORTED, "tree deeper than %d levels", ZHA_MAX_LEVELS);
    for (int l = 0; l < L; ++l)
        if (!(c->p[l] > 0.f) || !std::isfinite(c->p[l])) return fail(ZHA_ERR_INVALID_ARG, "p[%d]=%g must be in (0, inf)", l, c->p[l]);
    return ZHA_OK;
}

float scale_of(const zha_config* c) { return c->scale > 0.f ? c->scale : 1.0f / std::sqrt(static_cast<float>(c->d)); }

int tree_layout(const zha_config* c, TreeLayout* t) {
    ZHA_TRY(validate(c));
    int64_t n[kMaxLevels];
    t->Lcap = tree_levels(c->N_cap, c->B, c->b, c->L_fixed, n);
    t->R = c->R;
    t->vsum = c->vsum;
    const int64_t slices = static_cast<int64_t>(c->batch) * c->Hkv;
    size_t off = 0;
    t->off_ntree = off;
    off = align256(off + sizeof(int32_t) * c->batch);
    t->off_qref = off;
    off = align256(off + sizeof(float) * static_cast<size_t>(c->Hkv) * t->Lcap * c->R * c->d);
    for (int l = 0; l < kMaxLevels; ++l) {
        t->ncap[l] = l < t->Lcap ? std::max<int64_t>(n[l], 1) : 0;
        t->off_khat[l] = off;
        off = align256(off + sizeof(float) * static_cast<size_t>(slices) * t->ncap[l] * c->R * c->d);
        t->off_bhat[l] = off;
        off = align256(off + sizeof(float) * static_cast<size_t>(slices) * t->ncap[l] * c->R);
        t->off_vhat[l] = off;
        if (c->vsum) off = align256(off + sizeof(float) * static_cast<size_t>(slices) * t->ncap[l] * c->d);
    }
    t->total = off;
    return ZHA_OK;
}

TreeDev tree_view(const TreeLayout& t, void* tree) {
    TreeDev v{};
    char* base = static_cast<char*>(tree);
    v.n_tree = reinterpret_cast<int32_t*>(base + t.off_ntree);
    v.qref = reinterpret_cast<float*>(base + t.off_qref);
    for (int l = 0; l < kMaxLevels; ++l) {
        v.khat[l] = reinterpret_cast<float*>(base + t.off_khat[l]);
        v.bhat[l] = reinterpret_cast<float*>(base + t.off_bhat[l]);
        v.vhat[l] = t.vsum && t.ncap[l] > 0 ? reinterpret_cast<float*>(base + t.off_vhat[l]) : nullptr;
        v.ncap[l] = t.ncap[l];
    }
    v.Lcap = t.Lcap;
    v.R = t.R;
    return v;
}

// The decode attention clears its own per-group merge counters when it finishes, so
// these must hold zero between calls.  They sit at the front of every workspace layout,
// decode and prefill alike, and no prefill call writes there: a workspace moves
// between decode and chunks of any length without being zeroed again.
size_t ws_counter_bytes(const zha_config* c) {
    return align256(sizeof(uint32_t) * static_cast<size_t>(c->batch) * c->Hkv);
}

int ws_layout(const zha_config* c, int n_q, const TreeLayout& t, WsLayout* w) {
    if (n_q != 1) return fail(ZHA_ERR_UNSUPPORTED, "n_q=%d: decode takes one query per sequence", n_q);
    const int64_t groups = static_cast<int64_t>(c->batch) * c->Hkv;
    const int64_t ctas = static_cast<int64_t>(c->batch) * c->Hq * n_q;
    const int G = c->Hq / c->Hkv;
    w->cand_cap = t.ncap[0] + c->b;
    w->par_cap = std::max<int64_t>(t.ncap[0], 1);
    w->kb_cap = (w->cand_cap + 31) / 32;
    w->sel_cap = std::max<int64_t>(t.ncap[0], 1);
    w->item_cap = t.ncap[0] * ((c->B + kAttRows - 1) / kAttRows) + 2 + (c->N_cap + kAttRows - 1) / kAttRows;
    w->words = (t.ncap[0] + 31) / 32;
    size_t off = 0;
    w->off_counters = off; off = align256(off + sizeof(uint32_t) * groups);
    w->off_scores = off;   off = align256(off + sizeof(float) * ctas * w->cand_cap);
    w->off_parents = off;  off = align256(off + sizeof(int32_t) * ctas * 2 * w->par_cap);
    w->off_sel = off;      off = align256(off + sizeof(int32_t) * ctas * w->sel_cap);
    w->off_count = off;    off = align256(off + sizeof(int32_t) * ctas);
    w->off_items = off;    off = align256(off + sizeof(int2) * groups * w->item_cap);
    w->off_nitems = off;   off = align256(off + sizeof(int32_t) * groups);
    w->off_ml = off;       off = align256(off + sizeof(float2) * groups * kSplitMax * G);
    w->off_acc = off;      off = align256(off + sizeof(float) * groups * kSplitMax * G * c->d);
    w->off_rows = off;     off = align256(off + sizeof(int32_t) * groups);
    w->off_cand = off;     off = align256(off + sizeof(int32_t) * ctas);
    w->off_scanned = off;  off = align256(off + sizeof(int32_t) * groups);
    w->off_ballot = off;   off = align256(off + sizeof(uint32_t) * ctas * 2 * w->kb_cap);
    w->off_pr_ml = off;    off = align256(off + (c->vsum ? sizeof(float2) * ctas : 0));
    w->off_pr_acc = off;   off = align256(off + (c->vsum ? sizeof(float) * ctas * c->d : 0));
    w->total = off;
    if (static_cast<size_t>(G) * w->words * 4 > 200 * 1024)
        return fail(ZHA_ERR_UNSUPPORTED, "N_cap too large for the on-chip union bitmap");
    return ZHA_OK;
}

template <typename P>
P* at(void* base, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(base) + off); }

struct DevInfo {
    int sms = 0;
    int smem_optin = 0;
};

int dev_info(DevInfo* info) {
    static std::mutex mu;
    static DevInfo cache[64];
    int dev = 0;
    ZHA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(ZHA_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lk(mu);
    if (cache[dev].sms == 0) {
        ZHA_CUDA(cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev));
        ZHA_CUDA(cudaDeviceGetAttribute(&cache[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    }
    *info = cache[dev];
    return ZHA_OK;
}

// The calling thread's current CUDA context (the driver entry point is looked up once
// through the runtime, so the library needs no link against the driver library).
int current_context(CUcontext* out) {
    using GetCtx = CUresult (*)(CUcontext*);
    static std::mutex mu;
    static GetCtx fn = nullptr;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!fn) {
            void* p = nullptr;
            cudaDriverEntryPointQueryResult q;
            ZHA_CUDA(cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q));
            if (q != cudaDriverEntryPointSuccess || !p) return fail(ZHA_ERR_CUDA, "cuCtxGetCurrent is not available");
            fn = reinterpret_cast<GetCtx>(p);
        }
    }
    if (fn(out) == CUDA_SUCCESS && *out) return ZHA_OK;
    int dev = 0;   // no context yet: binding the current device initialises its primary context
    ZHA_CUDA(cudaGetDevice(&dev));
    ZHA_CUDA(cudaSetDevice(dev));
    if (fn(out) != CUDA_SUCCESS || !*out) return fail(ZHA_ERR_CUDA, "no current CUDA context");
    return ZHA_OK;
}

// Lets `kernel` use the device's opt-in shared memory (once per kernel, device and
// context: a device reset creates a new context, which starts with the defaults).
template <typename Kern>
int allow_smem(Kern kernel, size_t need) {
    static std::mutex mu;
    static std::map<std::pair<const void*, std::pair<int, CUcontext>>, size_t> done;   // -> dynamic smem allowed
    int dev = 0;
    ZHA_CUDA(cudaGetDevice(&dev));
    CUcontext ctx = nullptr;
    ZHA_TRY(current_context(&ctx));
    const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), std::make_pair(dev, ctx));
    size_t dyn_max = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = done.find(key);
        if (it != done.end()) dyn_max = it->second;
    }
    if (dyn_max == 0) {   // first launch of this kernel on this device
        DevInfo di;
        ZHA_TRY(dev_info(&di));
        cudaFuncAttributes fa;
        ZHA_CUDA(cudaFuncGetAttributes(&fa, kernel));
        dyn_max = static_cast<size_t>(di.smem_optin) - fa.sharedSizeBytes;
        ZHA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn_max)));
        std::lock_guard<std::mutex> lk(mu);
        done[key] = dyn_max;
    }
    if (need > dyn_max)
        return fail(ZHA_ERR_UNSUPPORTED, "kernel needs %zu B of dynamic shared memory (device max %zu)", need, dyn_max);
    return ZHA_OK;
}

int check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZHA_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    return ZHA_OK;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------- build / append
template <typename T, int D>
int run_build(const zha_config* c, const TreeLayout& lay, const void* K, const void* V, const int32_t* N, void* tree,
              cudaStream_t st) {
    BuildArgs a{};
    a.tree = tree_view(lay, tree);
    a.K = K;
    a.V = V;
    a.N = N;
    a.batch = c->batch; a.Hkv = c->Hkv; a.B = c->B; a.b = c->b; a.L_fixed = c->L_fixed;
    a.N_cap = c->N_cap;
    a.scale = scale_of(c);
    const int64_t slices = static_cast<int64_t>(c->batch) * c->Hkv;
    build_set_count_kernel<<<static_cast<unsigned>(cdiv(c->batch, 128)), 128, 0, st>>>(a.tree, N, c->batch, c->N_cap);
    ZHA_TRY(check_launch("build_set_count"));
    build_leaf_kernel<T, D><<<static_cast<unsigned>(cdiv(slices * lay.ncap[0] * lay.R * 32, 256)), 256, 0, st>>>(a);
    ZHA_TRY(check_launch("build_leaf"));
    for (int l = 2; l <= lay.Lcap; ++l) {
        build_upper_kernel<D><<<static_cast<unsigned>(cdiv(slices * lay.ncap[l - 1] * lay.R * 32, 256)), 256, 0, st>>>(a, l);
        ZHA_TRY(check_launch("build_upper"));
    }
    return ZHA_OK;
}

// Extension: leaves and ancestors that change, then the new count (the kernels read the old one).
template <typename T, int D>
int run_extend(const zha_config* c, const TreeLayout& lay, const void* K, const void* V, const int32_t* N, void* tree,
               cudaStream_t st) {
    BuildArgs a{};
    a.tree = tree_view(lay, tree);
    a.K = K;
    a.V = V;
    a.N = N;
    a.batch = c->batch; a.Hkv = c->Hkv; a.B = c->B; a.b = c->b; a.L_fixed = c->L_fixed;
    a.incremental = 1;
    a.N_cap = c->N_cap;
    a.scale = scale_of(c);
    const int64_t slices = static_cast<int64_t>(c->batch) * c->Hkv;
    build_leaf_kernel<T, D><<<static_cast<unsigned>(cdiv(slices * lay.ncap[0] * lay.R * 32, 256)), 256, 0, st>>>(a);
    ZHA_TRY(check_launch("extend_leaf"));
    for (int l = 2; l <= lay.Lcap; ++l) {
        build_upper_kernel<D><<<static_cast<unsigned>(cdiv(slices * lay.ncap[l - 1] * lay.R * 32, 256)), 256, 0, st>>>(a, l);
        ZHA_TRY(check_launch("extend_upper"));
    }
    extend_set_count_kernel<<<static_cast<unsigned>(cdiv(c->batch, 128)), 128, 0, st>>>(a.tree, N, c->batch, c->N_cap);
    return check_launch("extend_set_count");
}

template <typename T, int D>
int run_append(const zha_config* c, const TreeLayout& lay, void* K, void* V, const void* kn, const void* vn,
               int32_t* N, void* tree, cudaStream_t st) {
    AppendArgs a{};
    a.tree = tree_view(lay, tree);
    a.K = K; a.V = V; a.k_new = kn; a.v_new = vn; a.N = N;
    a.batch = c->batch; a.Hkv = c->Hkv; a.B = c->B; a.b = c->b; a.L_fixed = c->L_fixed;
    a.N_cap = c->N_cap;
    a.scale = scale_of(c);
    append_kernel<T, D><<<c->batch, 32 * c->Hkv, 0, st>>>(a);
    return check_launch("append");
}

// ---------------------------------------------------------------- route
PlanArgs plan_args(const zha_config* c, const WsLayout& wl, const TreeLayout& lay, const void* tree,
                   const int32_t* N, const int32_t* sel, const int32_t* cnt, int32_t sel_cap, void* ws);

// The plan region of the fused route: the G plan bitmaps (wl.words words each), then the
// bitmap of kept nodes of every level l >= 2 (for the count of distinct nodes read).
// Returns its words and fills the level offsets.
int route_region_words(const zha_config* c, const TreeLayout& lay, const WsLayout& wl, int* lvl_off) {
    const int G = c->Hq / c->Hkv;
    int64_t words = static_cast<int64_t>(G) * std::max<int64_t>(wl.words, 1);
    for (int l = 0; l < kMaxLevels; ++l) lvl_off[l] = 0;
    for (int l = 2; l <= lay.Lcap; ++l) {
        lvl_off[l - 1] = static_cast<int>(words);
        words += (lay.ncap[l - 1] + 31) / 32;
    }
    return static_cast<int>(std::min<int64_t>(words, int64_t{1} << 30));
}

// The route kernel builds the plan itself (clusters of G CTAs) when its plan region fits
// next to the router's shared memory on this device.
bool plan_fits_route(const zha_config* c, const TreeLayout& lay, const WsLayout& wl) {
    DevInfo di;
    if (dev_info(&di) != ZHA_OK) return false;
    int lvl_off[kMaxLevels];
    const size_t need = sizeof(RouteSmem) + 4 * static_cast<size_t>(route_region_words(c, lay, wl, lvl_off));
    return need + 1024 <= static_cast<size_t>(di.smem_optin);
}

// The cluster's CTAs help each other with levels too large for shared memory where that can
// pay: clusters (the plan fused) that leave at least half the SMs idle, over trees whose leaf
// level alone exceeds the router's shared score buffer.
bool route_help_pays(const RouteArgs& a, int ctas, int G) {
    DevInfo di;
    if (!a.fuse_plan || G < 2 || a.tree.R > 1 || a.pr_ml || dev_info(&di) != ZHA_OK) return false;
    return 2 * ctas <= di.sms && a.tree.ncap[0] > kScoresSmem;
}

template <typename T, int D, int NVR>
int run_route_t(const RouteArgs& a, int ctas, int G, cudaStream_t st) {
    auto kern = a.tree.R > 1 ? route_decode_kernel<T, D, NVR, true>
                : a.pr_ml ? route_decode_kernel<T, D, NVR, false, true>
                : route_help_pays(a, ctas, G) ? route_decode_kernel<T, D, NVR, false, false, true>
                : route_decode_kernel<T, D, NVR, false>;
    const size_t smem = sizeof(RouteSmem) + (a.fuse_plan ? 4 * static_cast<size_t>(a.region_words) : 0);
    ZHA_TRY(allow_smem(kern, smem));
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(static_cast<unsigned>(ctas));
    lc.blockDim = dim3(kRouteThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.fuse_plan ? static_cast<unsigned>(G) : 1u;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    ZHA_CUDA(cudaLaunchKernelEx(&lc, kern, a));
    return check_launch("route");
}

template <typename T, int D>
int run_route(const zha_config* c, const TreeLayout& lay, const WsLayout& wl, const void* tree, const void* Q,
              const int32_t* N, int32_t* sel, int32_t* cnt, int32_t sel_cap, void* ws, bool fuse, cudaStream_t st) {
    RouteArgs a{};
    a.tree = tree_view(lay, const_cast<void*>(tree));
    a.Q = Q; a.N = N; a.sel = sel; a.sel_count = cnt;
    a.cand = at<int32_t>(ws, wl.off_cand);
    a.ws_scores = at<float>(ws, wl.off_scores);
    a.ws_parents = at<int32_t>(ws, wl.off_parents);
    a.ws_ballot = at<uint32_t>(ws, wl.off_ballot);
    a.cand_cap = wl.cand_cap; a.par_cap = wl.par_cap; a.kb_cap = wl.kb_cap; a.N_cap = c->N_cap;
    a.sel_cap = sel_cap; a.batch = c->batch; a.Hq = c->Hq; a.Hkv = c->Hkv; a.B = c->B; a.b = c->b;
    a.L_fixed = c->L_fixed; a.n_q = 1;
    a.scale = scale_of(c);
    for (int l = 0; l < kMaxLevels; ++l) a.p[l] = c->p[l];
    a.plan = plan_args(c, wl, lay, tree, N, sel, cnt, sel_cap, ws);
    a.scanned = at<int32_t>(ws, wl.off_scanned);
    a.region_words = route_region_words(c, lay, wl, a.lvl_off);
    a.pr_ml = c->vsum ? at<float2>(ws, wl.off_pr_ml) : nullptr;
    a.pr_acc = c->vsum ? at<float>(ws, wl.off_pr_acc) : nullptr;
    a.fuse_plan = fuse ? 1 : 0;
    const int ctas = c->batch * c->Hq;
    const int G = c->Hq / c->Hkv;
    if (c->b <= 4) return run_route_t<T, D, 4>(a, ctas, G, st);
    if (c->b <= 8) return run_route_t<T, D, 8>(a, ctas, G, st);
    if (c->b <= 16) return run_route_t<T, D, 16>(a, ctas, G, st);
    return run_route_t<T, D, 32>(a, ctas, G, st);
}

// ---------------------------------------------------------------- attend
int make_kv_map(const zha_config* c, const void* base, CUtensorMap* map);
int make_q_map(const zha_config* c, const void* base, int64_t rows, CUtensorMap* map);

int attend_grid(const DevInfo& di) { return std::min(di.sms, kSplitMax); }   // a group has at most `grid` partials

// The tensor-core decode attention takes bf16, d = 128 and leaf blocks of whole 64-key
// tiles (items then start on a block and a 64-key box holds each); other shapes, or
// more groups than its shared memory holds, run on attend_kernel.
bool attend_tc_fits(const zha_config* c, const DevInfo& di) {
    return c->dtype == ZHA_BF16 && c->d == 128 && c->B % 64 == 0 &&
           tc_smem_bytes(c->batch * c->Hkv, attend_grid(di)) <= static_cast<size_t>(di.smem_optin);
}

template <int G>
int run_attend_tc(const zha_config* c, const AttendArgs& a, cudaStream_t st) {
    CUtensorMap mk, mv, mq;
    ZHA_TRY(make_kv_map(c, a.K, &mk));
    ZHA_TRY(make_kv_map(c, a.V, &mv));
    ZHA_TRY(make_q_map(c, a.Q, static_cast<int64_t>(c->batch) * a.n_q * c->Hq, &mq));
    auto kern = attend_tc_kernel<G>;
    DevInfo di;
    ZHA_TRY(dev_info(&di));
    const int grid = attend_grid(di);
    const size_t smem = tc_smem_bytes(a.groups, grid);
    ZHA_TRY(allow_smem(kern, smem));
    kern<<<grid, kTCThreads, smem, st>>>(mk, mv, mq, a);
    return check_launch("attend_tc");
}

template <typename T, int D, int G>
int run_attend_t(const AttendArgs& a, cudaStream_t st) {
    auto kern = attend_kernel<T, D, G>;
    const size_t smem = sizeof(AttSmem<T, D, G>) + sizeof(int) * (a.groups + 1);
    ZHA_TRY(allow_smem(kern, smem));
    DevInfo di;
    ZHA_TRY(dev_info(&di));
#ifndef ZHA_ATT_CTAS_PER_SM
#define ZHA_ATT_CTAS_PER_SM 1
#endif
    const int grid = std::min(ZHA_ATT_CTAS_PER_SM * di.sms, kSplitMax);   // a group has at most `grid` partials
    kern<<<grid, kAttThreads, smem, st>>>(a);
    return check_launch("attend");
}

template <typename T, int D>
int run_attend(const zha_config* c, const WsLayout& wl, const void* K, const void* V, const void* Q, float* O,
               void* ws, cudaStream_t st) {
    AttendArgs a{};
    a.K = K; a.V = V; a.Q = Q; a.O = O;
    a.items = at<int2>(ws, wl.off_items);
    a.n_items = at<int32_t>(ws, wl.off_nitems);
    a.part_ml = at<float2>(ws, wl.off_ml);
    a.part_acc = at<float>(ws, wl.off_acc);
    a.counters = at<uint32_t>(ws, wl.off_counters);
    a.pr_ml = c->vsum ? at<float2>(ws, wl.off_pr_ml) : nullptr;
    a.pr_acc = c->vsum ? at<float>(ws, wl.off_pr_acc) : nullptr;
    a.item_cap = wl.item_cap; a.N_cap = c->N_cap;
    a.groups = c->batch * c->Hkv; a.Hq = c->Hq; a.Hkv = c->Hkv; a.n_q = 1;
    a.qscale = scale_of(c) * 1.4426950408889634f;
    a.wait_ns = kWaitLongNs;
    DevInfo di;
    ZHA_TRY(dev_info(&di));
    if (attend_tc_fits(c, di)) {
        a.wait_ns = g_wait_ns.load();
        switch (c->Hq / c->Hkv) {
            case 1: return run_attend_tc<1>(c, a, st);
            case 2: return run_attend_tc<2>(c, a, st);
            default: return run_attend_tc<4>(c, a, st);
        }
    }
    switch (c->Hq / c->Hkv) {
        case 1: return run_attend_t<T, D, 1>(a, st);
        case 2: return run_attend_t<T, D, 2>(a, st);
        default: return run_attend_t<T, D, 4>(a, st);
    }
}

PlanArgs plan_args(const zha_config* c, const WsLayout& wl, const TreeLayout& lay, const void* tree,
                   const int32_t* N, const int32_t* sel, const int32_t* cnt, int32_t sel_cap, void* ws) {
    PlanArgs a{};
    a.sel = sel; a.sel_count = cnt; a.N = N;
    a.n_tree = tree_view(lay, const_cast<void*>(tree)).n_tree;
    a.items = at<int2>(ws, wl.off_items);
    a.n_items = at<int32_t>(ws, wl.off_nitems);
    a.rows = at<int32_t>(ws, wl.off_rows);
    a.item_cap = wl.item_cap; a.N_cap = c->N_cap;
    a.sel_cap = sel_cap; a.Hq = c->Hq; a.Hkv = c->Hkv; a.G = c->Hq / c->Hkv; a.B = c->B; a.n_q = 1;
    a.words = std::max<int64_t>(wl.words, 1);
    return a;
}


int run_plan(const zha_config* c, const WsLayout& wl, const TreeLayout& lay, const void* tree, const int32_t* N,
             const int32_t* sel, const int32_t* cnt, int32_t sel_cap, void* ws, cudaStream_t st) {
    const PlanArgs a = plan_args(c, wl, lay, tree, N, sel, cnt, sel_cap, ws);
    const size_t smem = sizeof(uint32_t) * a.G * a.words;
    ZHA_TRY(allow_smem(plan_decode_kernel, smem));
    plan_decode_kernel<<<c->batch * c->Hkv, kPlanThreads, smem, st>>>(a);
    return check_launch("plan");
}

// ---------------------------------------------------------------- chunked prefill (n_q > 1)
// Workspace of the prefill calls: route spill areas, the superblock plan, the
// partials of every row and the accounting counters.
struct PfLayout {
    int64_t slices, R, rows, cand_cap, par_cap, nJ_cap, item_cap, n1_cap, pair_cap;
    int64_t ucap;              // upper nodes scored on the tensor cores per row (0: that path is off)
    int up_off[kMaxLevels];
    int chunk_cap;             // 64-node chunks of the upper levels, at most
    size_t off_up, off_split, off_sbias;
    size_t off_spill_sc, off_spill_par, off_cand, off_totals, off_hdr, off_ctr, off_row_cnt, off_row_pairs, off_row_off;
    size_t off_jcount, off_jcur, off_pairs, off_items, off_tail_ml, off_tail_o, off_sel_ml, off_sel_o, off_steps;
    size_t total;
};

int pf_layout(const zha_config* c, int n_q, const TreeLayout& t, PfLayout* p) {
    if (n_q < 2) return fail(ZHA_ERR_INVALID_ARG, "n_q=%d", n_q);
    if (c->vsum) return fail(ZHA_ERR_UNSUPPORTED, "n_q=%d: chunked prefill does not take value summaries (vsum = 1)", n_q);
    if (c->dtype != ZHA_BF16) return fail(ZHA_ERR_UNSUPPORTED, "n_q=%d: chunked prefill takes bf16 K, V and Q", n_q);
    if (c->B != 64) return fail(ZHA_ERR_UNSUPPORTED, "n_q=%d: chunked prefill needs leaf blocks of B = 64 keys", n_q);
    const int G = c->Hq / c->Hkv;
    p->n1_cap = std::max<int64_t>(t.ncap[0], 1);
    if (p->n1_cap > (int64_t{kBitmapWords} * 32) * kPairsPerRow)
        return fail(ZHA_ERR_UNSUPPORTED, "chunked prefill: N_cap=%lld gives more than %d leaf blocks",
                    (long long)c->N_cap, kBitmapWords * 32 * kPairsPerRow);
    p->slices = static_cast<int64_t>(c->batch) * c->Hkv;
    p->R = static_cast<int64_t>(n_q) * G;
    p->rows = p->slices * p->R;
    if (p->rows * kPairsPerRow > (int64_t{1} << 31) - 1)
        return fail(ZHA_ERR_UNSUPPORTED, "chunked prefill: batch * n_q * Hq = %lld rows is too many", (long long)p->rows);
    p->cand_cap = t.ncap[0] + c->b;
    p->par_cap = std::max<int64_t>(t.ncap[0], 1);
    p->nJ_cap = (p->n1_cap + 3) / 4 + 1;
    p->pair_cap = p->rows * kPairsPerRow;
    p->item_cap = p->slices * ((p->R * kPairsPerRow + kTileRows - 1) / kTileRows + p->nJ_cap);
    const size_t D = static_cast<size_t>(c->d);
    size_t off = ws_counter_bytes(c);
    p->off_spill_sc = off;  off = align256(off + sizeof(float) * kPRSpillWarps * p->cand_cap);
    p->off_spill_par = off; off = align256(off + sizeof(int32_t) * kPRSpillWarps * 2 * p->par_cap);
    p->off_cand = off;      off = align256(off + sizeof(int32_t) * p->rows);
    p->off_totals = off;    off = align256(off + sizeof(unsigned long long) * p->slices * kSBOpts);
    p->off_steps = off;     off = align256(off + sizeof(int32_t) * p->slices);
    p->off_hdr = off;       off = align256(off + sizeof(int32_t) * 8);
    p->off_ctr = off;       off = align256(off + sizeof(int32_t) * 2);
    p->off_row_cnt = off;   off = align256(off + sizeof(int32_t) * p->rows);
    p->off_row_pairs = off; off = align256(off + sizeof(int32_t) * p->rows);
    p->off_row_off = off;   off = align256(off + sizeof(int32_t) * p->rows);
    p->off_jcount = off;    off = align256(off + sizeof(int32_t) * p->slices * p->nJ_cap);
    p->off_jcur = off;      off = align256(off + sizeof(int32_t) * p->slices * p->nJ_cap);
    p->off_pairs = off;     off = align256(off + sizeof(int4) * p->pair_cap);
    p->off_items = off;     off = align256(off + sizeof(int4) * p->item_cap);
    p->off_tail_ml = off;   off = align256(off + sizeof(float2) * p->rows);
    p->off_tail_o = off;    off = align256(off + sizeof(float) * p->rows * D);
    p->off_sel_ml = off;    off = align256(off + sizeof(float2) * p->pair_cap);
    p->off_sel_o = off;     off = align256(off + sizeof(float) * p->pair_cap * D);
    // the upper levels' scores of every row, computed on the tensor cores (R = 1, at least two
    // levels, at most kSUMaxCols upper nodes): column up_off[l-1] + node for level l >= 2
    p->ucap = 0;
    p->chunk_cap = 0;
    for (int l = 0; l < kMaxLevels; ++l) p->up_off[l] = 0;
    if (t.R == 1 && t.Lcap >= 2) {
        int64_t u = 0;
        int ch = 0;
        for (int l = 2; l <= t.Lcap; ++l) {
            p->up_off[l - 1] = static_cast<int>(u);
            u += t.ncap[l - 1];
            ch += static_cast<int>((t.ncap[l - 1] + kSUNodes - 1) / kSUNodes);
        }
        if (u <= kSUMaxCols) {
            p->ucap = u;
            p->chunk_cap = ch;
        }
    }
    const size_t tile_bytes = (c->d == 128 ? SULayout<128>::kBBytes : SULayout<64>::kBBytes);
    p->off_up = off;        off = align256(off + sizeof(float) * p->rows * p->ucap);
    p->off_split = off;     off = align256(off + tile_bytes * p->slices * p->chunk_cap);
    p->off_sbias = off;     off = align256(off + sizeof(float) * kSUNodes * p->slices * p->chunk_cap);
    p->total = off;
    return ZHA_OK;
}

// Tiled TMA map over K or V viewed as [batch*Hkv][N_cap][d] bf16, boxes of 64 keys x 64
// columns with the 128-byte swizzle the tensor-core operands expect.
int tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        ZHA_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
        if (q != cudaDriverEntryPointSuccess || !fn) return fail(ZHA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = encode;
    return ZHA_OK;
}

// bf16 K or V cache [batch*Hkv][N_cap][d] as boxes of 64 dims x 64 keys, 128-byte swizzle.
int make_kv_map(const zha_config* c, const void* base, CUtensorMap* map) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    ZHA_TRY(tensor_map_encoder(&encode));
    if (reinterpret_cast<uintptr_t>(base) % 16) return fail(ZHA_ERR_INVALID_ARG, "K/V must be 16-byte aligned");
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(c->d), static_cast<cuuint64_t>(c->N_cap),
                                static_cast<cuuint64_t>(c->batch) * c->Hkv};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(c->d) * 2, static_cast<cuuint64_t>(c->N_cap) * c->d * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ZHA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ZHA_OK;
}

// bf16 queries [rows][d] as boxes of 64 dims x 16 rows, 128-byte swizzle.
int make_q_map(const zha_config* c, const void* base, int64_t rows, CUtensorMap* map) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    ZHA_TRY(tensor_map_encoder(&encode));
    if (reinterpret_cast<uintptr_t>(base) % 16) return fail(ZHA_ERR_INVALID_ARG, "Q must be 16-byte aligned");
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(c->d), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(c->d) * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                              estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(ZHA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return ZHA_OK;
}

// The upper levels' scores of every chunk row on the tensor cores (score_upper_kernel).
template <int D>
int run_score_upper(const zha_config* c, const TreeLayout& lay, const PfLayout& pl, const void* tree, const void* Q,
                    int n_q, const int32_t* N, void* ws, cudaStream_t st) {
    SUArgs s{};
    s.Q = static_cast<const uint16_t*>(Q);
    s.tree = tree_view(lay, const_cast<void*>(tree));
    s.N = N;
    s.up = at<float>(ws, pl.off_up);
    s.split = at<unsigned char>(ws, pl.off_split);
    s.bias = at<float>(ws, pl.off_sbias);
    s.chunk_cap = pl.chunk_cap;
    s.ucap = pl.ucap;
    s.N_cap = c->N_cap;
    for (int l = 0; l < kMaxLevels; ++l) s.up_off[l] = pl.up_off[l];
    s.n_q = n_q; s.Hq = c->Hq; s.Hkv = c->Hkv; s.G = c->Hq / c->Hkv; s.B = c->B; s.b = c->b; s.L_fixed = c->L_fixed;
    s.R = static_cast<int>(pl.R);
    s.slices = static_cast<int>(pl.slices);
    s.tiles = static_cast<int>((pl.R + kSUTileRows - 1) / kSUTileRows);
    s.scale = scale_of(c);
    split_upper_kernel<D><<<static_cast<unsigned>(s.slices * s.chunk_cap), 256, 0, st>>>(s);
    ZHA_TRY(check_launch("split_upper"));
    auto kern = score_upper_kernel<D>;
    ZHA_TRY(allow_smem(kern, SULayout<D>::kSmem));
    kern<<<static_cast<unsigned>(s.slices * s.tiles), kSUThreads, SULayout<D>::kSmem, st>>>(s);
    return check_launch("score_upper");
}

template <int D, int NVR>
int run_proute_t(const PRouteArgs& a, int64_t rows, cudaStream_t st) {
    auto kern = a.tree.R > 1 ? route_prefill_kernel<uint16_t, D, NVR, true> : route_prefill_kernel<uint16_t, D, NVR, false>;
    ZHA_TRY(allow_smem(kern, sizeof(PRouteSmem)));
    DevInfo di;
    ZHA_TRY(dev_info(&di));
    const int64_t want = (rows + kPRWarps - 1) / kPRWarps;
    const int grid = static_cast<int>(std::min<int64_t>({want, 2 * di.sms, kPRSpillWarps / kPRWarps}));
    kern<<<grid, kPRThreads, sizeof(PRouteSmem), st>>>(a);
    return check_launch("route_prefill");
}

template <int D>
int run_proute(const zha_config* c, const TreeLayout& lay, const PfLayout& pl, const void* tree, const void* Q,
               int n_q, const int32_t* N, int32_t* sel, int32_t* cnt, int32_t sel_cap, void* ws, cudaStream_t st) {
    PRouteArgs a{};
    a.tree = tree_view(lay, const_cast<void*>(tree));
    a.Q = Q; a.N = N; a.sel = sel; a.sel_count = cnt;
    a.cand = at<int32_t>(ws, pl.off_cand);
    a.spill_sc = at<float>(ws, pl.off_spill_sc);
    a.spill_par = at<int32_t>(ws, pl.off_spill_par);
    a.cand_cap = pl.cand_cap; a.par_cap = pl.par_cap; a.N_cap = c->N_cap;
    a.sel_cap = sel_cap; a.batch = c->batch; a.Hq = c->Hq; a.Hkv = c->Hkv; a.B = c->B; a.b = c->b;
    a.L_fixed = c->L_fixed; a.n_q = n_q;
    a.scale = scale_of(c);
    for (int l = 0; l < kMaxLevels; ++l) a.p[l] = c->p[l];
    if (pl.ucap > 0) {   // the upper levels on the tensor cores first
        ZHA_TRY(run_score_upper<D>(c, lay, pl, tree, Q, n_q, N, ws, st));
        a.up = at<float>(ws, pl.off_up);
        a.ucap = pl.ucap;
        for (int l = 0; l < kMaxLevels; ++l) a.up_off[l] = pl.up_off[l];
    }
    const int64_t rows = static_cast<int64_t>(c->batch) * n_q * c->Hq;
    if (c->b <= 4) return run_proute_t<D, 4>(a, rows, st);
    if (c->b <= 8) return run_proute_t<D, 8>(a, rows, st);
    if (c->b <= 16) return run_proute_t<D, 16>(a, rows, st);
    return run_proute_t<D, 32>(a, rows, st);
}

PAttnArgs pattn_args(const zha_config* c, const PfLayout& pl, const TreeLayout& lay, const void* tree, const void* Q,
                     int n_q, const int32_t* N, const int32_t* sel, const int32_t* cnt, int32_t sel_cap, float* O,
                     void* ws, int dense) {
    PAttnArgs a{};
    a.Q = Q; a.O = O; a.N = N;
    a.n_tree = tree ? tree_view(lay, const_cast<void*>(tree)).n_tree : nullptr;
    a.sel = sel; a.sel_cap = sel_cap;
    a.row_cnt = at<int32_t>(ws, pl.off_row_cnt);
    a.pairs = at<int4>(ws, pl.off_pairs);
    a.items = at<int4>(ws, pl.off_items);
    a.hdr = at<int32_t>(ws, pl.off_hdr);
    a.ctr = at<int32_t>(ws, pl.off_ctr);
    a.tail_ml = at<float2>(ws, pl.off_tail_ml);
    a.tail_o = at<float>(ws, pl.off_tail_o);
    a.sel_ml = at<float2>(ws, pl.off_sel_ml);
    a.sel_o = at<float>(ws, pl.off_sel_o);
    a.steps = at<int32_t>(ws, pl.off_steps);
    a.N_cap = c->N_cap; a.item_cap = pl.item_cap;
    a.n_q = n_q; a.Hq = c->Hq; a.Hkv = c->Hkv; a.G = c->Hq / c->Hkv; a.B = c->B;
    a.R = static_cast<int>(pl.R); a.slices = static_cast<int>(pl.slices);
    a.tiles = static_cast<int>((pl.R + kTileRows - 1) / kTileRows);
    a.dense = dense;
    a.qscale = scale_of(c) * 1.4426950408889634f;
    return a;
}

template <int D>
int run_pattn_t(const zha_config* c, const PAttnArgs& a, const void* K, const void* V, cudaStream_t st) {
    CUtensorMap mk, mv;
    ZHA_TRY(make_kv_map(c, K, &mk));
    ZHA_TRY(make_kv_map(c, V, &mv));
    auto kern = attend_prefill_kernel<D>;
    ZHA_TRY(allow_smem(kern, PAttnLayout<D>::kSmem));
    DevInfo di;
    ZHA_TRY(dev_info(&di));
    kern<<<2 * di.sms, kPAThreads, PAttnLayout<D>::kSmem, st>>>(mk, mv, a);
    return check_launch("attend_prefill");
}

// The pair totals, step counters, plan header and item counters sit side by side and
// start every chunk at zero, whatever an earlier call with another n_q (hence another
// layout of the same workspace) left in these bytes.
int pf_reset(const PfLayout& pl, void* ws, cudaStream_t st) {
    ZHA_CUDA(cudaMemsetAsync(static_cast<char*>(ws) + pl.off_totals, 0,
                             pl.off_ctr + sizeof(int32_t) * 2 - pl.off_totals, st));
    return ZHA_OK;
}

int run_pattn(const zha_config* c, const PAttnArgs& a, const void* K, const void* V, cudaStream_t st) {
    return c->d == 128 ? run_pattn_t<128>(c, a, K, V, st) : run_pattn_t<64>(c, a, K, V, st);
}

// Plan + tensor-core attention + merge of a prefill chunk.
int run_prefill_attend(const zha_config* c, const TreeLayout& lay, const PfLayout& pl, const void* K, const void* V,
                       const void* tree, const void* Q, int n_q, const int32_t* N, const int32_t* sel,
                       const int32_t* cnt, int32_t sel_cap, float* O, void* ws, cudaStream_t st) {
    PPlanArgs p{};
    p.sel = sel; p.sel_count = cnt;
    p.n_tree = tree_view(lay, const_cast<void*>(tree)).n_tree;
    p.totals = at<unsigned long long>(ws, pl.off_totals);
    p.hdr = at<int32_t>(ws, pl.off_hdr);
    p.row_cnt = at<int32_t>(ws, pl.off_row_cnt);
    p.row_pairs = at<int32_t>(ws, pl.off_row_pairs);
    p.row_off = at<int32_t>(ws, pl.off_row_off);
    p.jcount = at<int32_t>(ws, pl.off_jcount);
    p.jcur = at<int32_t>(ws, pl.off_jcur);
    p.pairs = at<int4>(ws, pl.off_pairs);
    p.items = at<int4>(ws, pl.off_items);
    p.nJ_cap = pl.nJ_cap; p.item_cap = pl.item_cap; p.n1_cap = pl.n1_cap;
    p.sel_cap = sel_cap; p.n_q = n_q; p.Hq = c->Hq; p.Hkv = c->Hkv; p.G = c->Hq / c->Hkv; p.B = c->B;
    p.R = static_cast<int>(pl.R); p.slices = static_cast<int>(pl.slices);
    const int chunks = static_cast<int>(pl.slices) * kPlanChunks;
    ZHA_TRY(pf_reset(pl, ws, st));
    prefill_count_kernel<<<chunks, 256, 0, st>>>(p);
    prefill_choose_kernel<<<1, 1024, 0, st>>>(p);
    prefill_pairs_kernel<<<chunks, 256, 0, st>>>(p);
    prefill_scan_kernel<<<static_cast<int>(pl.slices), 1024, 0, st>>>(p);
    prefill_scatter_kernel<<<chunks, 256, 0, st>>>(p);
    ZHA_TRY(check_launch("prefill plan"));
    const PAttnArgs a = pattn_args(c, pl, lay, tree, Q, n_q, N, sel, cnt, sel_cap, O, ws, 0);
    ZHA_TRY(run_pattn(c, a, K, V, st));
    PMergeArgs m{};
    m.O = O;
    m.tail_ml = a.tail_ml; m.tail_o = a.tail_o; m.sel_ml = a.sel_ml; m.sel_o = a.sel_o;
    m.row_pairs = p.row_pairs; m.row_off = p.row_off;
    m.n_q = n_q; m.Hq = c->Hq; m.Hkv = c->Hkv; m.G = a.G; m.R = a.R; m.rows = pl.rows;
    const unsigned grid = static_cast<unsigned>((pl.rows * 32 + 255) / 256);
    if (c->d == 128) merge_prefill_kernel<128><<<grid, 256, 0, st>>>(m);
    else merge_prefill_kernel<64><<<grid, 256, 0, st>>>(m);
    return check_launch("merge_prefill");
}

int pf_setup(const zha_config* cfg, int n_q, TreeLayout* t, PfLayout* p, const void* ws, size_t ws_bytes) {
    ZHA_TRY(tree_layout(cfg, t));
    ZHA_TRY(pf_layout(cfg, n_q, *t, p));
    if (!ws) return fail(ZHA_ERR_INVALID_ARG, "ws is null");
    if (ws_bytes < p->total) return fail(ZHA_ERR_WORKSPACE, "workspace of %zu B < %zu B needed", ws_bytes, p->total);
    return ZHA_OK;
}

// Dispatch on (dtype, d).
#define ZHA_DISPATCH(c, FN, ...)                                                          \
    ((c)->dtype == ZHA_BF16 ? ((c)->d == 128 ? FN<uint16_t, 128>(__VA_ARGS__) : FN<uint16_t, 64>(__VA_ARGS__)) \
                            : ((c)->d == 128 ? FN<float, 128>(__VA_ARGS__) : FN<float, 64>(__VA_ARGS__)))

int need(const void* p, const char* name) {
    return p ? ZHA_OK : fail(ZHA_ERR_INVALID_ARG, "%s is null", name);
}

int check_ws(const WsLayout& wl, const void* ws, size_t ws_bytes) {
    ZHA_TRY(need(ws, "ws"));
    if (ws_bytes < wl.total) return fail(ZHA_ERR_WORKSPACE, "workspace of %zu B < %zu B needed", ws_bytes, wl.total);
    return ZHA_OK;
}

}  // namespace

// ---------------------------------------------------------------- allocation-free attention
// Scratch of zha_attend_noalloc: one file-scope device array, loaded with the
// library on every GPU that uses it and kept until the process exits.  All
// calls on a device share it; a call leaves its contents behind.
constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch in the current device's current context,
// looked up once per (device, context) with that device current (the symbol's
// host-side name is not a device address).  Keying on the context as well means a
// device reset, which gives the device a new primary context and reloads the
// library's module there, never leaves a stale address behind.
int noalloc_scratch_ptr(void** out) {
    static std::mutex mu;
    static std::map<std::pair<int, CUcontext>, void*> ptrs;
    int dev = 0;
    ZHA_CUDA(cudaGetDevice(&dev));
    CUcontext ctx = nullptr;
    ZHA_TRY(current_context(&ctx));
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair(dev, ctx);
    auto it = ptrs.find(key);
    if (it == ptrs.end()) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(ZHA_ERR_CUDA, "cudaGetSymbolAddress(g_noalloc_scratch): %s", cudaGetErrorString(e));
        it = ptrs.emplace(key, p).first;
    }
    *out = it->second;
    return ZHA_OK;
}

}  // namespace

// ======================================================================== C ABI
extern "C" {

int zha_levels_cap(const zha_config* cfg, int32_t* levels) {
    TreeLayout t;
    ZHA_TRY(need(levels, "levels"));
    ZHA_TRY(tree_layout(cfg, &t));
    *levels = t.Lcap;
    return ZHA_OK;
}

int zha_tree_bytes(const zha_config* cfg, size_t* bytes) {
    TreeLayout t;
    ZHA_TRY(need(bytes, "bytes"));
    ZHA_TRY(tree_layout(cfg, &t));
    *bytes = t.total;
    return ZHA_OK;
}

int zha_tree_level(const zha_config* cfg, int32_t level, size_t* khat_offset, size_t* bhat_offset,
                   int64_t* nodes_cap) {
    TreeLayout t;
    ZHA_TRY(need(khat_offset, "khat_offset"));
    ZHA_TRY(need(bhat_offset, "bhat_offset"));
    ZHA_TRY(need(nodes_cap, "nodes_cap"));
    ZHA_TRY(tree_layout(cfg, &t));
    if (level < 1 || level > t.Lcap) return fail(ZHA_ERR_INVALID_ARG, "level=%d outside 1..%d", level, t.Lcap);
    *khat_offset = t.off_khat[level - 1];
    *bhat_offset = t.off_bhat[level - 1];
    *nodes_cap = t.ncap[level - 1];
    return ZHA_OK;
}

int zha_tree_level_v(const zha_config* cfg, int32_t level, size_t* vhat_offset) {
    TreeLayout t;
    ZHA_TRY(need(vhat_offset, "vhat_offset"));
    ZHA_TRY(tree_layout(cfg, &t));
    if (!cfg->vsum) return fail(ZHA_ERR_INVALID_ARG, "the tree holds no value summaries (vsum = 0)");
    if (level < 1 || level > t.Lcap) return fail(ZHA_ERR_INVALID_ARG, "level=%d outside 1..%d", level, t.Lcap);
    *vhat_offset = t.off_vhat[level - 1];
    return ZHA_OK;
}

int zha_tree_count_offset(const zha_config* cfg, size_t* offset) {
    TreeLayout t;
    ZHA_TRY(need(offset, "offset"));
    ZHA_TRY(tree_layout(cfg, &t));
    *offset = t.off_ntree;
    return ZHA_OK;
}

int zha_workspace_bytes(const zha_config* cfg, int32_t n_q, size_t* bytes) {
    TreeLayout t;
    WsLayout w;
    ZHA_TRY(need(bytes, "bytes"));
    ZHA_TRY(tree_layout(cfg, &t));
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_layout(cfg, n_q, t, &p));
        *bytes = p.total;
        return ZHA_OK;
    }
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    *bytes = w.total;
    return ZHA_OK;
}

int zha_workspace_stats(const zha_config* cfg, int32_t n_q, size_t* rows_offset, size_t* cand_offset,
                        size_t* scanned_offset) {
    TreeLayout t;
    WsLayout w;
    ZHA_TRY(need(rows_offset, "rows_offset"));
    ZHA_TRY(need(cand_offset, "cand_offset"));
    ZHA_TRY(need(scanned_offset, "scanned_offset"));
    ZHA_TRY(tree_layout(cfg, &t));
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_layout(cfg, n_q, t, &p));
        *rows_offset = p.off_steps;
        *cand_offset = p.off_cand;
        *scanned_offset = p.off_cand;
        return ZHA_OK;
    }
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    *rows_offset = w.off_rows;
    *cand_offset = w.off_cand;
    *scanned_offset = w.off_scanned;
    return ZHA_OK;
}

int zha_attend_kernel(const zha_config* cfg, int32_t n_q, int32_t* kind) {
    TreeLayout t;
    ZHA_TRY(need(kind, "kind"));
    ZHA_TRY(tree_layout(cfg, &t));
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_layout(cfg, n_q, t, &p));
        *kind = 2;
        return ZHA_OK;
    }
    WsLayout w;
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    DevInfo di;
    ZHA_TRY(dev_info(&di));
    *kind = attend_tc_fits(cfg, di) ? 1 : 0;
    return ZHA_OK;
}

int zha_workspace_init(const zha_config* cfg, void* ws, size_t ws_bytes, zha_stream_t stream) {
    TreeLayout t;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(need(ws, "ws"));
    if (ws_bytes < ws_counter_bytes(cfg))
        return fail(ZHA_ERR_WORKSPACE, "workspace of %zu B < %zu B", ws_bytes, ws_counter_bytes(cfg));
    ZHA_CUDA(cudaMemsetAsync(ws, 0, ws_bytes, stream));
    return ZHA_OK;
}

int zha_build(const zha_config* cfg, const void* K, const void* V, const float* Qref, const int32_t* N, void* tree,
              zha_stream_t stream) {
    Range nvtx_range("zha_build");
    TreeLayout t;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(need(K, "K"));
    if (cfg->vsum) ZHA_TRY(need(V, "V (vsum = 1)"));
    ZHA_TRY(need(Qref, "Qref"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(tree, "tree"));
    const size_t qbytes = sizeof(float) * static_cast<size_t>(cfg->Hkv) * t.Lcap * cfg->R * cfg->d;
    ZHA_CUDA(cudaMemcpyAsync(static_cast<char*>(tree) + t.off_qref, Qref, qbytes, cudaMemcpyDeviceToDevice, stream));
    return ZHA_DISPATCH(cfg, run_build, cfg, t, K, V, N, tree, stream);
}

int zha_extend(const zha_config* cfg, const void* K, const void* V, const int32_t* N, void* tree,
               zha_stream_t stream) {
    Range nvtx_range("zha_extend");
    TreeLayout t;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(need(K, "K"));
    if (cfg->vsum) ZHA_TRY(need(V, "V (vsum = 1)"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(tree, "tree"));
    return ZHA_DISPATCH(cfg, run_extend, cfg, t, K, V, N, tree, stream);
}

int zha_append(const zha_config* cfg, void* K, void* V, const void* k_new, const void* v_new, int32_t* N,
               void* tree, zha_stream_t stream) {
    Range nvtx_range("zha_append");
    TreeLayout t;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(need(K, "K"));
    ZHA_TRY(need(V, "V"));
    ZHA_TRY(need(k_new, "k_new"));
    ZHA_TRY(need(v_new, "v_new"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(tree, "tree"));
    return ZHA_DISPATCH(cfg, run_append, cfg, t, K, V, k_new, v_new, N, tree, stream);
}

int zha_route(const zha_config* cfg, const void* tree, const void* Q, int32_t n_q, const int32_t* N, int32_t* sel,
              int32_t* sel_count, int32_t sel_cap, void* ws, size_t ws_bytes, zha_stream_t stream) {
    Range nvtx_range("zha_route");
    TreeLayout t;
    WsLayout w;
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_setup(cfg, n_q, &t, &p, ws, ws_bytes));
        ZHA_TRY(need(tree, "tree"));
        ZHA_TRY(need(Q, "Q"));
        ZHA_TRY(need(N, "N"));
        ZHA_TRY(need(sel, "sel"));
        ZHA_TRY(need(sel_count, "sel_count"));
        if (sel_cap < 1) return fail(ZHA_ERR_INVALID_ARG, "sel_cap=%d", sel_cap);
        return cfg->d == 128 ? run_proute<128>(cfg, t, p, tree, Q, n_q, N, sel, sel_count, sel_cap, ws, stream)
                             : run_proute<64>(cfg, t, p, tree, Q, n_q, N, sel, sel_count, sel_cap, ws, stream);
    }
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    ZHA_TRY(check_ws(w, ws, ws_bytes));
    ZHA_TRY(need(tree, "tree"));
    ZHA_TRY(need(Q, "Q"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(sel, "sel"));
    ZHA_TRY(need(sel_count, "sel_count"));
    if (sel_cap < 1) return fail(ZHA_ERR_INVALID_ARG, "sel_cap=%d", sel_cap);
    const bool fuse = plan_fits_route(cfg, t, w);
    if (!fuse) ZHA_CUDA(cudaMemsetAsync(at<int32_t>(ws, w.off_scanned), 0, sizeof(int32_t) * cfg->batch * cfg->Hkv, stream));
    ZHA_TRY(ZHA_DISPATCH(cfg, run_route, cfg, t, w, tree, Q, N, sel, sel_count, sel_cap, ws, fuse, stream));
    return fuse ? ZHA_OK : run_plan(cfg, w, t, tree, N, sel, sel_count, sel_cap, ws, stream);
}

int zha_attend(const zha_config* cfg, const void* K, const void* V, const void* tree, const void* Q, int32_t n_q,
               const int32_t* N, const int32_t* sel, const int32_t* sel_count, int32_t sel_cap, float* O, void* ws,
               size_t ws_bytes, zha_stream_t stream) {
    Range nvtx_range("zha_attend");
    TreeLayout t;
    WsLayout w;
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_setup(cfg, n_q, &t, &p, ws, ws_bytes));
        ZHA_TRY(need(K, "K"));
        ZHA_TRY(need(V, "V"));
        ZHA_TRY(need(tree, "tree"));
        ZHA_TRY(need(Q, "Q"));
        ZHA_TRY(need(N, "N"));
        ZHA_TRY(need(O, "O"));
        ZHA_TRY(need(sel, "sel (n_q > 1 takes the selection lists)"));
        ZHA_TRY(need(sel_count, "sel_count"));
        if (sel_cap < 1) return fail(ZHA_ERR_INVALID_ARG, "sel_cap=%d", sel_cap);
        return run_prefill_attend(cfg, t, p, K, V, tree, Q, n_q, N, sel, sel_count, sel_cap, O, ws, stream);
    }
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    ZHA_TRY(check_ws(w, ws, ws_bytes));
    ZHA_TRY(need(K, "K"));
    ZHA_TRY(need(V, "V"));
    ZHA_TRY(need(tree, "tree"));
    ZHA_TRY(need(Q, "Q"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(O, "O"));
    if (sel) {   // plan the gather from the given lists; else reuse the plan zha_route left in ws
        ZHA_TRY(need(sel_count, "sel_count"));
        if (sel_cap < 1) return fail(ZHA_ERR_INVALID_ARG, "sel_cap=%d", sel_cap);
        ZHA_TRY(run_plan(cfg, w, t, tree, N, sel, sel_count, sel_cap, ws, stream));
    }
    return ZHA_DISPATCH(cfg, run_attend, cfg, w, K, V, Q, O, ws, stream);
}

int zha_attend_noalloc(const zha_config* cfg, const void* K, const void* V, const void* tree, const void* Q,
                       int32_t n_q, const int32_t* N, const int32_t* sel, const int32_t* sel_count, int32_t sel_cap,
                       float* O, zha_stream_t stream) {
    Range nvtx_range("zha_attend_noalloc");
    if (n_q != 1)
        return fail(ZHA_ERR_UNSUPPORTED, "zha_attend_noalloc: decode only (n_q = 1, got %d); a chunked prefill "
                    "needs zha_attend with a workspace", n_q);
    if (cfg && cfg->vsum)
        return fail(ZHA_ERR_UNSUPPORTED, "zha_attend_noalloc: value summaries need the router's workspace (vsum = 1)");
    TreeLayout t;
    WsLayout w;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    if (w.total > kNoAllocScratchBytes)
        return fail(ZHA_ERR_WORKSPACE,
                    "zha_attend_noalloc: this configuration needs %zu B of scratch; the library's static scratch "
                    "holds %zu B (use zha_attend with a workspace)", w.total, kNoAllocScratchBytes);
    ZHA_TRY(need(K, "K"));
    ZHA_TRY(need(V, "V"));
    ZHA_TRY(need(tree, "tree"));
    ZHA_TRY(need(Q, "Q"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(sel, "sel"));
    ZHA_TRY(need(sel_count, "sel_count"));
    ZHA_TRY(need(O, "O"));
    if (sel_cap < 1) return fail(ZHA_ERR_INVALID_ARG, "sel_cap=%d", sel_cap);
    void* ws = nullptr;
    ZHA_TRY(noalloc_scratch_ptr(&ws));
    // the per-group merge counters must start at zero; everything else is written before it is read
    ZHA_CUDA(cudaMemsetAsync(static_cast<char*>(ws) + w.off_counters, 0,
                             sizeof(uint32_t) * static_cast<size_t>(cfg->batch) * cfg->Hkv, stream));
    ZHA_TRY(run_plan(cfg, w, t, tree, N, sel, sel_count, sel_cap, ws, stream));
    return ZHA_DISPATCH(cfg, run_attend, cfg, w, K, V, Q, O, ws, stream);
}

int zha_decode(const zha_config* cfg, void* K, void* V, void* tree, const void* q, const void* k_new,
               const void* v_new, int32_t* N, float* O, void* ws, size_t ws_bytes, zha_stream_t stream) {
    Range nvtx_range("zha_decode");
    TreeLayout t;
    WsLayout w;
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(ws_layout(cfg, 1, t, &w));
    ZHA_TRY(check_ws(w, ws, ws_bytes));
    ZHA_TRY(need(q, "q"));
    ZHA_TRY(need(O, "O"));
    ZHA_TRY(zha_append(cfg, K, V, k_new, v_new, N, tree, stream));
    int32_t* sel = at<int32_t>(ws, w.off_sel);
    int32_t* cnt = at<int32_t>(ws, w.off_count);
    const int32_t sel_cap = static_cast<int32_t>(w.sel_cap);
    const bool fuse = plan_fits_route(cfg, t, w);
    if (!fuse) ZHA_CUDA(cudaMemsetAsync(at<int32_t>(ws, w.off_scanned), 0, sizeof(int32_t) * cfg->batch * cfg->Hkv, stream));
    ZHA_TRY(ZHA_DISPATCH(cfg, run_route, cfg, t, w, tree, q, N, sel, cnt, sel_cap, ws, fuse, stream));
    if (!fuse) ZHA_TRY(run_plan(cfg, w, t, tree, N, sel, cnt, sel_cap, ws, stream));
    return ZHA_DISPATCH(cfg, run_attend, cfg, w, K, V, q, O, ws, stream);
}

int zha_dense(const zha_config* cfg, const void* K, const void* V, const void* Q, int32_t n_q, const int32_t* N,
              float* O, void* ws, size_t ws_bytes, zha_stream_t stream) {
    Range nvtx_range("zha_dense");
    TreeLayout t;
    WsLayout w;
    if (n_q > 1) {
        PfLayout p;
        ZHA_TRY(pf_setup(cfg, n_q, &t, &p, ws, ws_bytes));
        ZHA_TRY(need(K, "K"));
        ZHA_TRY(need(V, "V"));
        ZHA_TRY(need(Q, "Q"));
        ZHA_TRY(need(N, "N"));
        ZHA_TRY(need(O, "O"));
        ZHA_TRY(pf_reset(p, const_cast<void*>(ws), stream));
        const PAttnArgs a = pattn_args(cfg, p, t, nullptr, Q, n_q, N, nullptr, nullptr, 0, O, ws, 1);
        return run_pattn(cfg, a, K, V, stream);
    }
    ZHA_TRY(tree_layout(cfg, &t));
    ZHA_TRY(ws_layout(cfg, n_q, t, &w));
    ZHA_TRY(check_ws(w, ws, ws_bytes));
    ZHA_TRY(need(K, "K"));
    ZHA_TRY(need(V, "V"));
    ZHA_TRY(need(Q, "Q"));
    ZHA_TRY(need(N, "N"));
    ZHA_TRY(need(O, "O"));
    plan_dense_kernel<<<cfg->batch * cfg->Hkv, 256, 0, stream>>>(N, at<int2>(ws, w.off_items), at<int32_t>(ws, w.off_nitems),
                                                                at<int32_t>(ws, w.off_rows), w.item_cap, cfg->N_cap,
                                                                cfg->Hkv, cfg->Hq / cfg->Hkv);
    ZHA_TRY(check_launch("plan_dense"));
    return ZHA_DISPATCH(cfg, run_attend, cfg, w, K, V, Q, O, ws, stream);
}

int zha_get_status(int32_t* status_bits, int32_t clear, zha_stream_t stream) {
    ZHA_TRY(need(status_bits, "status_bits"));
    ZHA_CUDA(cudaStreamSynchronize(stream));
    int v = 0;
    ZHA_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof v));
    if (clear) {
        const int z = 0;
        ZHA_CUDA(cudaMemcpyToSymbol(g_status, &z, sizeof z));
    }
    *status_bits = v;
    return ZHA_OK;
}

int zha_set_wait_limit(uint64_t ns, uint64_t* previous) {
    const uint64_t old = g_wait_ns.exchange(ns);
    if (previous) *previous = old;
    return ZHA_OK;
}

const char* zha_last_error(void) { return g_err; }

}  // extern "C"
