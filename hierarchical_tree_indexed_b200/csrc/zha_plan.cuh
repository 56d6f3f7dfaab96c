// zha_plan.cuh -- the gather plan of decode attention: per (sequence, KV head),
// the ascending union of the blocks selected by its G query heads, each with the
// mask of the heads that need it, plus the current chunk and the sink.
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: I(q) = {0} u (union of the kept level-1
// chunks) u C_cur(q); the first token is the sink ([EoQ] "Zyphra Hierarchical
// Attention: The End of Quadratic Attention?", How the tree is built and searched).
#pragma once

#include "zha_common.cuh"

namespace zha {

constexpr int kPlanThreads = 512;
constexpr int kItemRowsMax = 64;   // rows of one item (and of one attention stage)

// item: x = first key, y = key count | head mask << 16
__device__ __forceinline__ int2 make_item(int64_t start, int count, uint32_t mask) {
    return make_int2(static_cast<int>(start), count | static_cast<int>(mask << 16));
}

struct PlanArgs {
    const int32_t* sel;        // [batch][n_q][Hq][sel_cap]
    const int32_t* sel_count;  // [batch][n_q][Hq]
    const int32_t* N;          // [batch]
    const int32_t* n_tree;     // [batch]
    int2* items;               // [groups][item_cap]
    int32_t* n_items;          // [groups]
    int32_t* rows;             // [groups] keys gathered (accounting)
    int64_t item_cap, N_cap;
    int sel_cap, Hq, Hkv, G, B, n_q;
    int64_t words;             // bitmap words per head: ceil(n1cap / 32)
};

// The gather plan of group g (one (sequence, KV head)), computed by one block of
// kPlanThreads threads.  bits: shared memory for G * a.words words; scan: kPlanThreads/32+1 ints.
__device__ void plan_group(const PlanArgs& a, int g, uint32_t* bits, int* scan) {
    const int s = g / a.Hkv, kv = g % a.Hkv, tid = threadIdx.x;
    const int G = a.G;
    const uint32_t all = (1u << G) - 1u;
    const int64_t N = a.N[s], Ntree = a.n_tree[s];
    if (N < 1 || N > a.N_cap || Ntree > N) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.n_items[g] = 0; a.rows[g] = 0; }
        __syncthreads();
        return;
    }
    const int64_t t = N - 1;
    const int64_t n1 = Ntree / a.B;
    const int64_t words = (n1 + 31) / 32;
    for (int h = 0; h < G; ++h)
        for (int i = tid; i < static_cast<int>(words); i += kPlanThreads) bits[h * a.words + i] = 0u;
    __syncthreads();
    // every head's selected blocks into its bitmap: counts first, then all entries at once
    __shared__ int s_cnt[8], s_off[9];
    if (tid < G) {
        const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + tid;
        s_cnt[tid] = min(__ldcg(&a.sel_count[row]), a.sel_cap);
    }
    __syncthreads();
    if (tid == 0) {
        s_off[0] = 0;
        for (int h = 0; h < G; ++h) s_off[h + 1] = s_off[h] + s_cnt[h];
    }
    __syncthreads();
    for (int j = tid; j < s_off[G]; j += kPlanThreads) {
        int h = 0;
        while (j >= s_off[h + 1]) ++h;
        const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + h;
        const int32_t blk = __ldcg(&a.sel[row * a.sel_cap + (j - s_off[h])]);
        if (blk >= 0 && blk < n1) atomicOr(&bits[h * a.words + (blk >> 5)], 1u << (blk & 31));
    }
    const int64_t cb = min(t / a.B, n1);   // C_cur = [cb*B, t]
    if (tid < G && cb < n1) atomicOr(&bits[tid * a.words + (cb >> 5)], 1u << (cb & 31));
    __syncthreads();
    // compaction of the union, ascending: thread owns words [w0, w1)
    const int64_t per = (words + kPlanThreads - 1) / kPlanThreads;
    const int64_t w0 = min(words, tid * per), w1 = min(words, w0 + per);
    const int nsplit = (a.B + kItemRowsMax - 1) / kItemRowsMax;   // items per block (B > 64)
    int c = 0;
    for (int64_t wd = w0; wd < w1; ++wd) {
        uint32_t o = 0;
        for (int h = 0; h < G; ++h) o |= bits[h * a.words + wd];
        c += __popc(o) * nsplit;
    }
    int total;
    int pos = block_exclusive_scan<kPlanThreads / 32>(c, scan, &total);
    int2* out = a.items + static_cast<int64_t>(g) * a.item_cap;
    for (int64_t wd = w0; wd < w1; ++wd) {
        uint32_t o = 0;
        for (int h = 0; h < G; ++h) o |= bits[h * a.words + wd];
        while (o) {
            const int bit = __ffs(o) - 1;
            o &= o - 1;
            uint32_t m = 0;
            for (int h = 0; h < G; ++h) m |= ((bits[h * a.words + wd] >> bit) & 1u) << h;
            if (nsplit == 1) {
                out[pos++] = make_item((wd * 32 + bit) * a.B, a.B, m);
            } else {
                for (int st = 0; st < a.B; st += kItemRowsMax)
                    out[pos++] = make_item((wd * 32 + bit) * a.B + st, min(kItemRowsMax, a.B - st), m);
            }
        }
    }
    if (tid == 0) {
        int n = total;
        int64_t rows = static_cast<int64_t>(nsplit == 1 ? total : total / nsplit) * a.B;
        if (n1 >= 1) {   // sink: key 0 for the heads whose block 0 is not in the union
            uint32_t m0 = 0;
            for (int h = 0; h < G; ++h) m0 |= (bits[h * a.words] & 1u) << h;
            if ((m0 & all) != all) { out[n++] = make_item(0, 1, all & ~m0); rows += 1; }
        }
        if (cb == n1)   // C_cur past the last leaf block: the keys [n1*B, t], 64 at a time
            for (int64_t st = cb * a.B; st <= t && n < a.item_cap; st += kItemRowsMax) {
                const int c = static_cast<int>(t - st + 1 < kItemRowsMax ? t - st + 1 : kItemRowsMax);
                out[n++] = make_item(st, c, all);
                rows += c;
            }
        a.n_items[g] = n;
        a.rows[g] = static_cast<int32_t>(rows);
    }
    __syncthreads();
}

// One CTA per (sequence, KV head).
__global__ void __launch_bounds__(kPlanThreads) plan_decode_kernel(PlanArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ int scan[kPlanThreads / 32 + 1];
    plan_group(a, blockIdx.x, reinterpret_cast<uint32_t*>(smem_raw), scan);
}

// Dense baseline plan: items of 64 keys covering [0, N) for every head.
__global__ void plan_dense_kernel(const int32_t* N, int2* items, int32_t* n_items, int32_t* rows,
                                  int64_t item_cap, int64_t N_cap, int Hkv, int G) {
    const int g = blockIdx.x, s = g / Hkv;
    const int64_t n = N[s];
    if (n < 1 || n > N_cap) {
        if (threadIdx.x == 0) { raise_status(ZHA_ERR_INVALID_ARG); n_items[g] = 0; rows[g] = 0; }
        return;
    }
    if (threadIdx.x == 0) rows[g] = static_cast<int32_t>(n);
    const int64_t cnt = (n + kItemRowsMax - 1) / kItemRowsMax;
    const uint32_t all = (1u << G) - 1u;
    for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x)
        items[g * item_cap + i] = make_item(i * kItemRowsMax, static_cast<int>(n - i * kItemRowsMax < kItemRowsMax ? n - i * kItemRowsMax : kItemRowsMax), all);
    if (threadIdx.x == 0) n_items[g] = static_cast<int32_t>(cnt);
}

}  // namespace zha
