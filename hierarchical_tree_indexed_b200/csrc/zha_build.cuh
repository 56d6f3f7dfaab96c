// zha_build.cuh -- tree construction and incremental append.
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Tree Construction (F_C, the tangent khat_r, bhat_r;
// upper levels "constructed recursively from their children's summaries");
// [EoQ] "Zyphra Hierarchical Attention: The End of Quadratic Attention?",
// A query's path ("the tree is built on the fly as the context grows").
//
// Every summary -- leaf block of raw keys, or upper node over child summaries
// -- is the tangent of a log-sum-exp at the level's reference query qhat:
//   z_i = scale * qhat . x_i + c_i      (c_i = 0 for raw keys, bhat of the child otherwise)
//   F   = LSE_i z_i,  khat = sum_i softmax(z)_i x_i,  bhat = F - scale * qhat . khat.
// One warp computes one summary with a streaming (online) softmax over 16-byte
// row loads; build and append call the same routine, so an appended tree is
// bitwise identical to a rebuilt one.  With R reference queries per node (planes
// r = 0..R-1), every plane of a node is its own tangent; above level 1 a child's
// estimate is its best plane, max_p (scale q.khat_p + bhat_p) (ties to the lower
// plane), and its pooled key is that plane's khat.
#pragma once

#include "zha_common.cuh"

namespace zha {

// One warp: summary of `count` rows (row stride D elements of T, 16-byte aligned),
// optional per-row bias (nullptr = 0), reference query q (fp32 [D]).  WV: the value
// rows vrows (same layout) are pooled with the same weights into vhat_out.
template <typename T, int D, bool WV = false>
__device__ void summarize_rows(const T* __restrict__ rows, const float* __restrict__ bias, int count,
                               const float* __restrict__ q, float scale, float* __restrict__ khat_out,
                               float* __restrict__ bhat_out, const T* __restrict__ vrows = nullptr,
                               float* __restrict__ vhat_out = nullptr) {
    constexpr int VEC = Elem<T>::kVec;   // elements per 16-byte load
    constexpr int LPR = D / VEC;         // lanes per row
    constexpr int RPW = 32 / LPR;        // rows per warp-wide load
    constexpr int U = 4;                 // loads in flight per lane
    static_assert(D % VEC == 0 && 32 % LPR == 0, "row must split evenly over the warp");
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;

    float qv[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) qv[e] = q[li * VEC + e] * scale;

    float m = -INFINITY, l = 0.f, acc[VEC], accv[WV ? VEC : 1];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
#pragma unroll
    for (int e = 0; e < (WV ? VEC : 1); ++e) accv[e] = 0.f;

    for (int base = 0; base < count; base += RPW * U) {
        float x[U][VEC], xv[U][WV ? VEC : 1], z[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int row = base + u * RPW + sub;
            if (row < count) {
                Elem<T>::load16(rows + static_cast<int64_t>(row) * D + li * VEC, x[u]);
                if constexpr (WV) Elem<T>::load16(vrows + static_cast<int64_t>(row) * D + li * VEC, xv[u]);
            } else {
#pragma unroll
                for (int e = 0; e < VEC; ++e) x[u][e] = 0.f;
                if constexpr (WV) {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) xv[u][e] = 0.f;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) s = fmaf(qv[e], x[u][e], s);
            z[u] = s;
        }
#pragma unroll
        for (int o = 1; o < LPR; o <<= 1)
#pragma unroll
            for (int u = 0; u < U; ++u) z[u] += __shfl_xor_sync(0xffffffffu, z[u], o);
        float mi = -INFINITY;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int row = base + u * RPW + sub;
            z[u] = row < count ? z[u] + (bias ? bias[row] : 0.f) : -INFINITY;
            mi = fmaxf(mi, z[u]);
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) mi = fmaxf(mi, __shfl_xor_sync(0xffffffffu, mi, o));
        const float mn = fmaxf(m, mi);              // finite: row `base` exists
        const float alpha = expf(m - mn);           // m = -inf -> 0
        float ws = 0.f, w[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            w[u] = expf(z[u] - mn);                 // padded rows -> 0
            ws += w[u];
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) ws += __shfl_xor_sync(0xffffffffu, ws, o);
        l = l * alpha + ws;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            float a = acc[e] * alpha;
#pragma unroll
            for (int u = 0; u < U; ++u) a = fmaf(w[u], x[u][e], a);
            acc[e] = a;
        }
        if constexpr (WV) {
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                float a = accv[e] * alpha;
#pragma unroll
                for (int u = 0; u < U; ++u) a = fmaf(w[u], xv[u][e], a);
                accv[e] = a;
            }
        }
        m = mn;
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    const float inv = 1.f / l;
    if constexpr (WV) {
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < VEC; ++e) accv[e] += __shfl_xor_sync(0xffffffffu, accv[e], o);
        if (sub == 0) {
#pragma unroll
            for (int e = 0; e < VEC; e += 4)
                *reinterpret_cast<float4*>(vhat_out + li * VEC + e) =
                    make_float4(accv[e] * inv, accv[e + 1] * inv, accv[e + 2] * inv, accv[e + 3] * inv);
        }
    }
    float pd = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        acc[e] *= inv;
        pd = fmaf(qv[e], acc[e], pd);
    }
#pragma unroll
    for (int o = 1; o < LPR; o <<= 1) pd += __shfl_xor_sync(0xffffffffu, pd, o);
    if (sub == 0) {
#pragma unroll
        for (int e = 0; e < VEC; e += 4)
            *reinterpret_cast<float4*>(khat_out + li * VEC + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        if (lane == 0) *bhat_out = m + logf(l) - pd;
    }
}

// One warp: the summary at reference query q of `cnt` children with R planes each
// (child c, plane p at kh[(c * R + p) * D], bh[c * R + p]): each child enters with
// its best plane's estimate and key.
template <int D>
__device__ void summarize_children_planes(const float* __restrict__ kh, const float* __restrict__ bh, int cnt,
                                          int R, const float* __restrict__ q, float scale,
                                          float* __restrict__ khat_out, float* __restrict__ bhat_out) {
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31;
    float qv[VF];
#pragma unroll
    for (int e = 0; e < VF; ++e) qv[e] = q[lane * VF + e] * scale;
    float m = -INFINITY, l = 0.f, acc[VF];
#pragma unroll
    for (int e = 0; e < VF; ++e) acc[e] = 0.f;
    for (int c = 0; c < cnt; ++c) {
        float best = -INFINITY;
        int bp = 0;
        for (int pl = 0; pl < R; ++pl) {
            float x[VF];
            load_n<float, VF>(kh + (static_cast<int64_t>(c) * R + pl) * D + lane * VF, x);
            float dd = 0.f;
#pragma unroll
            for (int e = 0; e < VF; ++e) dd = fmaf(qv[e], x[e], dd);
            const float t = warp_sum(dd) + bh[static_cast<int64_t>(c) * R + pl];
            if (t > best) { best = t; bp = pl; }
        }
        float x[VF];
        load_n<float, VF>(kh + (static_cast<int64_t>(c) * R + bp) * D + lane * VF, x);
        const float mn = fmaxf(m, best);
        const float alpha = expf(m - mn);
        const float wgt = expf(best - mn);
        l = l * alpha + wgt;
#pragma unroll
        for (int e = 0; e < VF; ++e) acc[e] = fmaf(wgt, x[e], acc[e] * alpha);
        m = mn;
    }
    const float inv = 1.f / l;
    float pd = 0.f;
#pragma unroll
    for (int e = 0; e < VF; ++e) {
        acc[e] *= inv;
        pd = fmaf(qv[e], acc[e], pd);
    }
    pd = warp_sum(pd);
#pragma unroll
    for (int e = 0; e < VF; ++e) khat_out[lane * VF + e] = acc[e];
    if (lane == 0) *bhat_out = m + logf(l) - pd;
}

struct BuildArgs {
    TreeDev tree;
    const void* K;      // [batch][Hkv][N_cap][d]
    const void* V;      // the same layout; read when the tree holds value summaries
    const int32_t* N;   // [batch]
    int batch, Hkv, B, b, L_fixed;
    int incremental;    // 1: the tree already indexes tree.n_tree[s] keys; summarise only what changes
    int64_t N_cap;
    float scale;
};

// Extending a tree from n_old to N keys changes the leaf blocks from floor(n_old/B)
// on, and at level l only their ancestors (node index = leaf index / b^(l-1)) and
// any level the old tree did not have.  Returns the first node of level l to redo.
__device__ __forceinline__ int64_t first_changed(int64_t n_old, int l, int B, int b, int L_fixed) {
    int64_t no[kMaxLevels];
    const int L_old = tree_levels(n_old, B, b, L_fixed, no);
    if (l > L_old) return 0;
    int64_t first = n_old / B;
    for (int k = 1; k < l; ++k) first /= b;
    return first;
}

// Level 1: one warp per (sequence, KV head, leaf block, plane).
template <typename T, int D>
__global__ void __launch_bounds__(256) build_leaf_kernel(BuildArgs a) {
    const int R = a.tree.R;
    const int64_t gw0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int pl = static_cast<int>(gw0 % R);
    const int64_t gw = gw0 / R;
    const int64_t n1cap = a.tree.ncap[0];
    const int64_t slice = gw / n1cap, j = gw % n1cap;
    if (slice >= static_cast<int64_t>(a.batch) * a.Hkv) return;
    const int s = static_cast<int>(slice / a.Hkv), h = static_cast<int>(slice % a.Hkv);
    const int64_t N = a.N[s];
    if (N < 0 || N > a.N_cap) {
        if (j == 0 && (threadIdx.x & 31) == 0) raise_status(ZHA_ERR_INVALID_ARG);
        return;
    }
    if (j >= N / a.B) return;
    if (a.incremental) {
        const int64_t n_old = a.tree.n_tree[s];
        if (N < n_old || j < n_old / a.B) return;   // shrinking is refused by the count kernel
    }
    const T* rows = static_cast<const T*>(a.K) + (slice * a.N_cap + j * a.B) * D;
    const float* q = a.tree.qref + (static_cast<int64_t>(h) * a.tree.Lcap * R + pl) * D;
    float* kh = a.tree.khat[0] + ((slice * n1cap + j) * R + pl) * D;
    float* bh = a.tree.bhat[0] + (slice * n1cap + j) * R + pl;
    if (a.tree.vhat[0]) {   // value summaries: R = 1
        const T* vrows = static_cast<const T*>(a.V) + (slice * a.N_cap + j * a.B) * D;
        summarize_rows<T, D, true>(rows, nullptr, a.B, q, a.scale, kh, bh, vrows,
                                   a.tree.vhat[0] + (slice * n1cap + j) * D);
    } else {
        summarize_rows<T, D>(rows, nullptr, a.B, q, a.scale, kh, bh);
    }
}

// Level l >= 2: one warp per (sequence, KV head, node) over its children at l-1.
template <int D>
__device__ __forceinline__ void summarize_node(const TreeDev& t, int64_t slice, int h, int l, int64_t i,
                                               int64_t n_child, int b, float scale, int pl = 0) {
    const int R = t.R;
    const int64_t c0 = i * b;
    const int cnt = static_cast<int>(min(static_cast<int64_t>(b), n_child - c0));
    const int64_t cc = t.ncap[l - 2];
    const float* rows = t.khat[l - 2] + (slice * cc + c0) * R * D;
    const float* bias = t.bhat[l - 2] + (slice * cc + c0) * R;
    const float* q = t.qref + ((static_cast<int64_t>(h) * t.Lcap + (l - 1)) * R + pl) * D;
    float* kh = t.khat[l - 1] + ((slice * t.ncap[l - 1] + i) * R + pl) * D;
    float* bh = t.bhat[l - 1] + (slice * t.ncap[l - 1] + i) * R + pl;
    if (R == 1 && t.vhat[l - 1])
        summarize_rows<float, D, true>(rows, bias, cnt, q, scale, kh, bh, t.vhat[l - 2] + (slice * cc + c0) * D,
                                       t.vhat[l - 1] + (slice * t.ncap[l - 1] + i) * D);
    else if (R == 1) summarize_rows<float, D>(rows, bias, cnt, q, scale, kh, bh);
    else summarize_children_planes<D>(rows, bias, cnt, R, q, scale, kh, bh);
}

template <int D>
__global__ void __launch_bounds__(256) build_upper_kernel(BuildArgs a, int l) {
    const int64_t gw0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int pl = static_cast<int>(gw0 % a.tree.R);
    const int64_t gw = gw0 / a.tree.R;
    const int64_t ncap = a.tree.ncap[l - 1];
    const int64_t slice = gw / ncap, i = gw % ncap;
    if (slice >= static_cast<int64_t>(a.batch) * a.Hkv) return;
    const int s = static_cast<int>(slice / a.Hkv), h = static_cast<int>(slice % a.Hkv);
    int64_t n[kMaxLevels];
    const int64_t N = a.N[s];
    if (N < 0 || N > a.N_cap) return;
    const int L = tree_levels(N, a.B, a.b, a.L_fixed, n);
    if (L < 0 || l > L || i >= n[l - 1]) return;
    if (a.incremental) {
        const int64_t n_old = a.tree.n_tree[s];
        if (N < n_old || i < first_changed(n_old, l, a.B, a.b, a.L_fixed)) return;
    }
    summarize_node<D>(a.tree, slice, h, l, i, n[l - 2], a.b, a.scale, pl);
}

__global__ void build_set_count_kernel(TreeDev t, const int32_t* N, int batch, int64_t N_cap) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s < batch) t.n_tree[s] = (N[s] >= 0 && N[s] <= N_cap) ? N[s] : 0;
}

// After an extension: the tree now indexes N[s] keys (a shorter N is refused).
__global__ void extend_set_count_kernel(TreeDev t, const int32_t* N, int batch, int64_t N_cap) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= batch) return;
    if (N[s] < t.n_tree[s] || N[s] > N_cap) raise_status(ZHA_ERR_INVALID_ARG);
    else t.n_tree[s] = N[s];
}

struct AppendArgs {
    TreeDev tree;
    void* K;
    void* V;
    const void* k_new;   // [batch][Hkv][d]
    const void* v_new;
    int32_t* N;          // [batch] cache lengths, incremented
    int batch, Hkv, B, b, L_fixed;
    int64_t N_cap;
    float scale;
};

// One CTA per sequence, one warp per KV head.  Writes the new token, then, if it
// completes a leaf block, summarises the block and its ancestor path; when the
// depth grows, the whole new top level is summarised.
template <typename T, int D>
__global__ void append_kernel(AppendArgs a) {
    const int s = blockIdx.x, h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ int s_ok;
    __shared__ int64_t s_N;
    if (threadIdx.x == 0) {
        const int64_t N = a.tree.n_tree[s];
        int ok = 1;
        if (N != a.N[s] || N < 0) { raise_status(ZHA_ERR_INVALID_ARG); ok = 0; }
        else if (N >= a.N_cap) { raise_status(ZHA_ERR_CAPACITY); ok = 0; }
        s_ok = ok;
        s_N = N;
    }
    __syncthreads();
    if (!s_ok) return;
    const int64_t N = s_N;
    if (h < a.Hkv) {
        const int64_t slice = static_cast<int64_t>(s) * a.Hkv + h;
        T* Kr = static_cast<T*>(a.K) + (slice * a.N_cap + N) * D;
        T* Vr = static_cast<T*>(a.V) + (slice * a.N_cap + N) * D;
        const T* kn = static_cast<const T*>(a.k_new) + slice * D;
        const T* vn = static_cast<const T*>(a.v_new) + slice * D;
        for (int e = lane; e < D; e += 32) {
            Kr[e] = kn[e];
            Vr[e] = vn[e];
        }
        const int64_t N1 = N + 1;
        if (N1 % a.B == 0) {
            __syncwarp();
            __threadfence_block();
            const int64_t j = N1 / a.B - 1;
            const int R = a.tree.R;
            const T* rows = static_cast<const T*>(a.K) + (slice * a.N_cap + j * a.B) * D;
            for (int pl = 0; pl < R; ++pl) {
                const float* q = a.tree.qref + (static_cast<int64_t>(h) * a.tree.Lcap * R + pl) * D;
                float* kh = a.tree.khat[0] + ((slice * a.tree.ncap[0] + j) * R + pl) * D;
                float* bh = a.tree.bhat[0] + (slice * a.tree.ncap[0] + j) * R + pl;
                if (a.tree.vhat[0])   // value summaries: R = 1
                    summarize_rows<T, D, true>(rows, nullptr, a.B, q, a.scale, kh, bh,
                                               static_cast<const T*>(a.V) + (slice * a.N_cap + j * a.B) * D,
                                               a.tree.vhat[0] + (slice * a.tree.ncap[0] + j) * D);
                else
                    summarize_rows<T, D>(rows, nullptr, a.B, q, a.scale, kh, bh);
            }
            int64_t n0[kMaxLevels], n1[kMaxLevels];
            const int L0 = tree_levels(N, a.B, a.b, a.L_fixed, n0);
            const int L1 = tree_levels(N1, a.B, a.b, a.L_fixed, n1);
            int64_t idx = j;
            for (int l = 2; l <= L1; ++l) {
                __syncwarp();
                __threadfence_block();
                idx /= a.b;
                if (l > L0) {
                    for (int64_t i = 0; i < n1[l - 1]; ++i) {
                        for (int pl = 0; pl < R; ++pl) summarize_node<D>(a.tree, slice, h, l, i, n1[l - 2], a.b, a.scale, pl);
                        __syncwarp();
                    }
                } else {
                    for (int pl = 0; pl < R; ++pl) summarize_node<D>(a.tree, slice, h, l, idx, n1[l - 2], a.b, a.scale, pl);
                }
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        a.tree.n_tree[s] = static_cast<int32_t>(N + 1);
        a.N[s] = static_cast<int32_t>(N + 1);
    }
}

}  // namespace zha
