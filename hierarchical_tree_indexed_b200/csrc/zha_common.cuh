// zha_common.cuh -- device helpers shared by the kernels of the tree-indexed
// sparse attention library (sm_100a): element loads, warp/block reductions,
// the tree geometry rule, the sticky status word, and thin PTX wrappers for
// mbarriers and 1-D bulk async copies (cp.async.bulk, no multicast).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "zha.h"

namespace zha {

constexpr int kMaxLevels = ZHA_MAX_LEVELS;

// Sticky device status: bit (1 << zha_status) for every error raised on the device.
__device__ int g_status;

__device__ __forceinline__ void raise_status(int code) { atomicOr(&g_status, 1 << code); }

// ---------------------------------------------------------------- geometry
// n_1 = floor(N/B) complete leaf blocks, n_{l+1} = ceil(n_l / b); the depth is
// the first level with at most b nodes, or L_fixed levels when L_fixed > 0
// ("Subquadratic Attention with a Hierarchical Tree-Structured Indexer",
// Tree Construction: a level-l node spans C^l keys, here B*b^(l-1)).
// Returns L, or -1 when more than kMaxLevels levels would be needed.
// N < 2^31 (zha_config's N_cap is bounded so), so the arithmetic is 32-bit: a 64-bit
// division is a long emulated sequence on the GPU, on every router's critical path.
__host__ __device__ inline int tree_levels(int64_t N, int B, int b, int L_fixed, int64_t* n) {
    uint32_t cur = static_cast<uint32_t>(N > 0 ? N : 0) / static_cast<uint32_t>(B);
    const uint32_t ub = static_cast<uint32_t>(b);
    int L = 1;
    n[0] = cur;
    while (L_fixed > 0 ? L < L_fixed : cur > ub) {
        if (L >= kMaxLevels) return -1;
        cur = (cur + ub - 1) / ub;
        n[L++] = cur;
    }
    return L;
}

// Device view of the tree buffer (built by the host from zha_config).
struct TreeDev {
    int32_t* n_tree;            // [batch] keys the tree indexes
    float* qref;                // [Hkv][Lcap][R][d]
    float* khat[kMaxLevels];    // level l-1: [batch][Hkv][ncap][R][d]
    float* bhat[kMaxLevels];    // level l-1: [batch][Hkv][ncap][R]
    float* vhat[kMaxLevels];    // level l-1: [batch][Hkv][ncap][d] value summaries (R = 1), or null
    int64_t ncap[kMaxLevels];
    int Lcap;
    int R;                      // reference queries (planes) per node
};

// ---------------------------------------------------------------- elements
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Elements per 16-byte vector and the loader of one vector as fp32.
template <typename T> struct Elem;
template <> struct Elem<float> {
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void load16(const float* p, float* out) {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
};
template <> struct Elem<uint16_t> {   // bf16 stored as its 16 bits
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void load16(const uint16_t* p, float* out) {
        uint4 v = *reinterpret_cast<const uint4*>(p);
        out[0] = bf16_lo(v.x); out[1] = bf16_hi(v.x); out[2] = bf16_lo(v.y); out[3] = bf16_hi(v.y);
        out[4] = bf16_lo(v.z); out[5] = bf16_hi(v.z); out[6] = bf16_lo(v.w); out[7] = bf16_hi(v.w);
    }
};

// n consecutive elements (n in {1,2,4,8}) starting at p, as fp32.
template <typename T, int n>
__device__ __forceinline__ void load_n(const T* p, float* out);
template <> __device__ __forceinline__ void load_n<float, 2>(const float* p, float* out) {
    float2 v = *reinterpret_cast<const float2*>(p); out[0] = v.x; out[1] = v.y;
}
template <> __device__ __forceinline__ void load_n<float, 4>(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p); out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <> __device__ __forceinline__ void load_n<uint16_t, 2>(const uint16_t* p, float* out) {
    uint32_t v = *reinterpret_cast<const uint32_t*>(p); out[0] = bf16_lo(v); out[1] = bf16_hi(v);
}
template <> __device__ __forceinline__ void load_n<uint16_t, 4>(const uint16_t* p, float* out) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    out[0] = bf16_lo(v.x); out[1] = bf16_hi(v.x); out[2] = bf16_lo(v.y); out[3] = bf16_hi(v.y);
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<uint16_t>(uint16_t x) {
    return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

// ---------------------------------------------------------------- warp / block
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ uint32_t warp_or(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v |= __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Exclusive prefix sum of one int per thread over the whole block (NW warps).
// scratch: >= NW+1 ints of shared memory.  Returns the prefix; *total gets the sum.
template <int NW>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[w] = x;
    __syncthreads();
    if (w == 0) {
        int t = lane < NW ? scratch[lane] : 0;
        int s = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < NW) scratch[lane] = s - t;
        if (lane == NW - 1) scratch[NW] = s;
    }
    __syncthreads();
    int r = scratch[w] + x - v;
    *total = scratch[NW];
    __syncthreads();
    return r;
}

// ---------------------------------------------------------------- PTX: mbarrier + bulk copy
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
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
// atomicAdd with acquire-release semantics at GPU scope; returns the old value.
__device__ __forceinline__ uint32_t atomic_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Non-blocking: whether the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// The bound of a wait on something that cannot fail to come: a copy this CTA issued
// itself, or the tensor cores' completion of its own MMAs (~2 s).
constexpr uint64_t kWaitLongNs = 2000000000ull;

// Waits for the phase with the given parity; gives up after limit_ns of %globaltimer and
// returns false.  limit_ns = 0 gives up at once unless the phase has already completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns = kWaitLongNs) {
    if (mbar_test_wait(bar, parity)) return true;
    if (limit_ns == 0) return false;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
    }
}
// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Split cluster barrier: every thread of every CTA of the cluster arrives (release), then
// waits (acquire) for all of them; shared-memory writes before the arrival, local or
// remote, are visible to every CTA of the cluster after the wait.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// The shared::cluster address of `p` (this CTA's shared memory) in the CTA of the given rank.
__device__ __forceinline__ uint32_t cluster_map(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}
// Atomic OR into a word of a cluster CTA's shared memory (no return value).
__device__ __forceinline__ void dsmem_or(uint32_t addr, uint32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.or.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// The shared::cluster address, in the CTA of the given rank, of this CTA's shared address a.
__device__ __forceinline__ uint32_t cluster_map_addr(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
__device__ __forceinline__ uint32_t dsmem_ld_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t dsmem_ld_acquire_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.acquire.cluster.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint64_t dsmem_ld_u64(uint32_t a) {
    uint64_t v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float dsmem_ld_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void dsmem_st_f32(uint32_t a, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void dsmem_st_release_u32(uint32_t a, uint32_t v) {
    asm volatile("st.release.cluster.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t dsmem_atom_add_u32(uint32_t a, uint32_t v) {
    uint32_t old;
    asm volatile("atom.relaxed.cluster.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void dsmem_red_add_release_u32(uint32_t a, uint32_t v) {
    asm volatile("red.release.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void dsmem_red_max_s32(uint32_t a, int v) {
    asm volatile("red.relaxed.cluster.shared::cluster.max.s32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace zha
