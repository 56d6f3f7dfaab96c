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
constexpr int kPlanSpec = 4;       // selection entries per thread loaded with the counts

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

// The gather plan of group g from the per-head bitmaps of its selected blocks, by one
// block of kPlanThreads threads.  bits: G bitmaps of a.words words in shared memory, word
// w of head h at bits[h * a.words + w], holding every selected block below n_1 = Ntree / B
// (bits at and beyond n_1 clear); the current chunk's block is added here.  scan:
// kPlanThreads/32+1 ints.  N, Ntree: the sequence's key count and tree count, valid
// (1 <= N <= N_cap, Ntree <= N).
struct NoTail {
    __device__ void operator()() const {}
};
// tail(): run by warp 1 while thread 0 writes the plan's last items (used for bookkeeping
// that does not touch the plan).
template <typename Tail = NoTail>
__device__ void plan_emit(const PlanArgs& a, int g, uint32_t* bits, int* scan, int64_t N, int64_t Ntree,
                          Tail tail = Tail()) {
    const int tid = threadIdx.x;
    const int G = a.G;
    const uint32_t all = (1u << G) - 1u;
    const int64_t t = N - 1;
    const uint32_t uB = static_cast<uint32_t>(a.B);   // keys < 2^31: 32-bit divisions
    const int64_t n1 = static_cast<uint32_t>(Ntree) / uB;
    const int64_t words = (n1 + 31) / 32;
    const int64_t cb = min(static_cast<int64_t>(static_cast<uint32_t>(t) / uB), n1);   // C_cur = [cb*B, t]
    if (tid < G && cb < n1) atomicOr(&bits[tid * a.words + (cb >> 5)], 1u << (cb & 31));
    __syncthreads();
    // compaction of the union, ascending.  Warp w takes the words [w*per, (w+1)*per), per a
    // multiple of 32: its lanes load 32 words at a time and count their blocks; one block scan
    // places the warps' runs; then each warp walks its non-empty words one at a time, a lane per
    // block (a word of a cluster often holds 32 blocks).
    const int nsplit = (a.B + kItemRowsMax - 1) / kItemRowsMax;   // items per block (B > 64)
    constexpr int NWP = kPlanThreads / 32;
    const int lane = tid & 31, wp = tid >> 5;
    int2* out = a.items + static_cast<int64_t>(g) * a.item_cap;
    const int64_t per = ((words + NWP - 1) / NWP + 31) / 32 * 32;
    const int64_t w0 = min(words, wp * per), w1 = min(words, w0 + per);
    auto word_union = [&](int64_t wd) {
        uint32_t o = 0;
        if (wd < w1)
            for (int hh = 0; hh < G; ++hh) o |= bits[hh * a.words + wd];
        return o;
    };
    int mine = 0;
    for (int64_t c = w0; c < w1; c += 32) mine += __popc(word_union(c + lane));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
    int total;
    int pos = block_exclusive_scan<NWP>(lane == 0 ? mine * nsplit : 0, scan, &total);
    pos = __shfl_sync(0xffffffffu, pos, 0);
    for (int64_t c = w0; c < w1; c += 32) {
        const uint32_t u = word_union(c + lane);
        const int cntw = __popc(u) * nsplit;
        int incl = cntw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        uint32_t nz = __ballot_sync(0xffffffffu, u != 0u);
        while (nz) {
            const int j = __ffs(nz) - 1;
            nz &= nz - 1u;
            const uint32_t oj = __shfl_sync(0xffffffffu, u, j);
            const int pj = pos + __shfl_sync(0xffffffffu, incl - cntw, j);
            const int64_t wj = c + j;
            if ((oj >> lane) & 1u) {
                uint32_t m = 0;
                for (int hh = 0; hh < G; ++hh) m |= ((bits[hh * a.words + wj] >> lane) & 1u) << hh;
                const int idx = pj + __popc(oj & ((1u << lane) - 1u)) * nsplit;
                const int64_t k0 = (wj * 32 + lane) * a.B;
                if (nsplit == 1) {
                    out[idx] = make_item(k0, a.B, m);
                } else {
                    for (int st = 0, k = 0; st < a.B; st += kItemRowsMax, ++k)
                        out[idx + k] = make_item(k0 + st, min(kItemRowsMax, a.B - st), m);
                }
            }
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
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
    } else if (tid >= 32 && tid < 64) {
        tail();
    }
    __syncthreads();
}

// The gather plan of group g (one (sequence, KV head)) from the selection lists in global
// memory, computed by one block of kPlanThreads threads.  bits: shared memory for
// G * a.words words; scan: kPlanThreads/32+1 ints.
__device__ void plan_group(const PlanArgs& a, int g, uint32_t* bits, int* scan) {
    const int s = g / a.Hkv, kv = g % a.Hkv, tid = threadIdx.x;
    const int G = a.G;
    const int64_t N = a.N[s];
    const int64_t Ntree = a.n_tree[s];
    if (N < 1 || N > a.N_cap || Ntree > N) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.n_items[g] = 0; a.rows[g] = 0; }
        __syncthreads();
        return;
    }
    const int64_t n1 = static_cast<uint32_t>(Ntree) / static_cast<uint32_t>(a.B);
    const int64_t words = (n1 + 31) / 32;
    // every head's selected blocks into its bitmap: kPlanThreads / G threads per head load
    // the head's count and their first kPlanSpec entries together (one round trip; entries
    // past the count are dropped), while the bitmaps are cleared
    const int tph = kPlanThreads / G, h = tid / tph, r = tid % tph;
    const int64_t hrow = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + (h < G ? h : 0);
    const int32_t* hsel = a.sel + hrow * a.sel_cap;
    int32_t spec[kPlanSpec];
#pragma unroll
    for (int k = 0; k < kPlanSpec; ++k) {
        const int j = r + k * tph;
        spec[k] = (h < G && j < a.sel_cap) ? __ldcg(&hsel[j]) : -1;
    }
    const int hcnt = h < G ? min(__ldcg(&a.sel_count[hrow]), a.sel_cap) : 0;
    for (int hh = 0; hh < G; ++hh)
        for (int i = tid; i < static_cast<int>(words); i += kPlanThreads) bits[hh * a.words + i] = 0u;
    __syncthreads();
    uint32_t* hb = bits + (h < G ? h : 0) * a.words;
#pragma unroll
    for (int k = 0; k < kPlanSpec; ++k) {
        const int32_t blk = spec[k];
        if (r + k * tph < hcnt && blk >= 0 && blk < n1) atomicOr(&hb[blk >> 5], 1u << (blk & 31));
    }
    for (int j = r + kPlanSpec * tph; j < hcnt; j += tph) {
        const int32_t blk = __ldcg(&hsel[j]);
        if (blk >= 0 && blk < n1) atomicOr(&hb[blk >> 5], 1u << (blk & 31));
    }
    __syncthreads();
    plan_emit(a, g, bits, scan, N, Ntree);
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
