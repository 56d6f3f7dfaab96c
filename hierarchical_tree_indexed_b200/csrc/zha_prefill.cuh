// zha_prefill.cuh -- chunked prefill: n_q causal queries per sequence over a
// tree built on the first N - n_q keys.
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing (top-p per level, the index set I(q) and
// o(q) = Attn(q, K_I, V_I)); [EoQ] "Zyphra Hierarchical Attention: The End of
// Quadratic Attention?" (the first token is the attention sink).  Query i of
// the chunk sits at t = N - n_q + i; the tree covers n_1 = floor((N - n_q)/B)
// blocks and C_cur(t) = [n_1 B, t] is the causal tail.
//
// Routing (route_prefill_kernel): one warp walks the tree for one (query,
// head): the children scan is the decode scan, the top-p cut is the same rule
// (fixed-point masses, ties to the lower id) found by a bisection over the
// score keys.  Selected block ids come out ascending.
//
// Attention runs on the tensor cores (tcgen05, accumulators in TMEM, K/V tiles
// by TMA) as work items of up to 128 query rows x a list of 64-key blocks:
//   tail items     -- 128 consecutive rows of one (sequence, KV head) over the
//                     causal tail [n_1 B, t], masked per row (query-major);
//   selected items -- the rows that selected any block of one superblock
//                     (SB aligned blocks), over the union of those blocks,
//                     masked per row (key-major: a block is loaded once for all
//                     the rows that picked it, since rows of one query tile
//                     rarely share blocks).
// Each item leaves a partial (running max m, sum l, unnormalised o) per row;
// a merge kernel combines a row's partials in a fixed order.  SB is the
// smallest power of two >= 4 whose partial count fits the workspace, chosen on
// the device.
#pragma once

#include <cuda_bf16.h>

#include "zha_common.cuh"
#include "zha_topp.cuh"
#include "zha_route.cuh"
#include "zha_umma.cuh"

namespace zha {

// ======================================================================== routing
constexpr int kPRThreads = 256;
constexpr int kPRWarps = kPRThreads / 32;
constexpr int kPRScores = 1536;     // per-warp candidate scores in shared memory
constexpr int kPRBins = kWarpCutBins;
constexpr int kPRMembers = kWarpCutMembers;
constexpr int kPRParents = 512;     // per-warp parent ids, per buffer
constexpr int kPRSpillWarps = 2 * 160 * kPRWarps;   // warps with a workspace spill area (grid cap)

struct PRouteArgs {
    TreeDev tree;
    const void* Q;          // [batch][n_q][Hq][d]
    const int32_t* N;       // [batch], keys including the chunk
    int32_t* sel;           // [batch][n_q][Hq][sel_cap]
    int32_t* sel_count;     // [batch][n_q][Hq]
    int32_t* cand;          // [batch][n_q][Hq] nodes scored (accounting)
    float* spill_sc;        // [kPRSpillWarps][cand_cap]
    int32_t* spill_par;     // [kPRSpillWarps][2][par_cap]
    const float* up;        // the upper levels' scores from score_upper_kernel, [slices][R][ucap]; or null
    int64_t ucap;
    int up_off[kMaxLevels]; // column of level l's node 0 (index l - 1), l >= 2
    int64_t cand_cap, par_cap, N_cap;
    int sel_cap, batch, Hq, Hkv, B, b, L_fixed, n_q;
    float scale;
    float p[kMaxLevels];
};

struct PRouteSmem {
    float sc[kPRWarps][kPRScores];
    int32_t par[kPRWarps][2][kPRParents];
    unsigned long long hist[kPRWarps][kPRBins];
    unsigned long long mem_key[kPRWarps][kPRMembers];   // (score key << 32) | ~slot of a member
    unsigned long long mem_mass[kPRWarps][kPRMembers];
};

// One warp per (sequence, query, query head) row, rows taken in a grid-stride loop.
template <typename T, int D, int NVR, bool MP>
__global__ void __launch_bounds__(kPRThreads, 2) route_prefill_kernel(PRouteArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    PRouteSmem& sm = *reinterpret_cast<PRouteSmem*>(smem_raw);
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int gw = blockIdx.x * kPRWarps + w;
    const int nw = gridDim.x * kPRWarps;
    const int G = a.Hq / a.Hkv;
    const int b = a.b;
    // rows < 2^31 (the workspace layout bounds batch * n_q * Hq far below that)
    const int rows = a.batch * a.n_q * a.Hq;
    const int per_seq = a.n_q * a.Hq;
    float* spill_sc = a.spill_sc + static_cast<int64_t>(gw) * a.cand_cap;
    int32_t* spill_par = a.spill_par + static_cast<int64_t>(gw) * 2 * a.par_cap;
    int cached_s = -1, L = 0;
    int64_t n[kMaxLevels];
    for (int x = gw; x < rows; x += nw) {
        const int s = x / per_seq;
        const int hq = x % a.Hq;
        const int64_t slice = static_cast<int64_t>(s) * a.Hkv + hq / G;
        const int64_t N = a.N[s];
        const int64_t Ntree = a.tree.n_tree[s];
        if (N < a.n_q || N > a.N_cap || Ntree != N - a.n_q) {
            if (lane == 0) {
                raise_status(ZHA_ERR_INVALID_ARG);
                a.sel_count[x] = 0;
                a.cand[x] = 0;
            }
            continue;
        }
        // the row's scores at the upper levels, when the tensor cores computed them
        const float* up_row = nullptr;
        if (a.up) {
            const int i = (x % per_seq) / a.Hq;
            up_row = a.up + (slice * (static_cast<int64_t>(a.n_q) * G) + static_cast<int64_t>(i) * G + hq % G) * a.ucap;
        }
        float qv[VF];
        load_n<T, VF>(static_cast<const T*>(a.Q) + static_cast<int64_t>(x) * D + lane * VF, qv);
#pragma unroll
        for (int e = 0; e < VF; ++e) qv[e] *= a.scale;
        if (s != cached_s) {   // the geometry of this sequence's tree, once per sequence
            L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
            cached_s = s;
        }
        int32_t* bufs[4] = {sm.par[w][0], sm.par[w][1], spill_par, spill_par + a.par_cap};
        int cur = 0;
        int np = static_cast<int>((n[L - 1] + b - 1) / b);
        if (np > kPRParents) cur = 2;
        for (int i = lane; i < np; i += 32) bufs[cur][i] = i;
        __syncwarp();
        int64_t scored = 0;
        for (int l = L; l >= 1 && np > 0; --l) {
            const int64_t nl = n[l - 1];
            const int nc = np * b;
            const int32_t* par = bufs[cur];
            const int64_t last_parent = (nl - 1) / b;
            scored += nc - (par[np - 1] == last_parent ? b - (nl - last_parent * b) : 0);
            float* sc = nc <= kPRScores ? sm.sc[w] : spill_sc;
            const int64_t ncap = a.tree.ncap[l - 1];
            const int R = MP ? a.tree.R : 1;
            const float* kh = a.tree.khat[l - 1] + slice * ncap * R * D;
            const float* bh = a.tree.bhat[l - 1] + slice * ncap * R;
            const bool read_up = up_row && l >= 2;
            if (read_up) {   // read, not scanned: the kept parents' children
                const float* us = up_row + a.up_off[l - 1];
                for (int i = lane; i < nc; i += 32) {
                    const int64_t c = static_cast<int64_t>(par[i / b]) * b + i % b;
                    sc[i] = c < nl ? __ldg(us + c) : -INFINITY;
                }
            }
            for (int pi = 0; pi < (read_up ? 0 : np); pi += 2) {
                const int64_t c0 = static_cast<int64_t>(par[pi]) * b;
                const int cnt0 = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
                if constexpr (!MP) {
                    if (pi + 1 < np) {
                        const int64_t c1 = static_cast<int64_t>(par[pi + 1]) * b;
                        const int cnt1 = static_cast<int>(min(static_cast<int64_t>(b), nl - c1));
                        scan_children2<D, NVR>(kh + c0 * D, bh + c0, cnt0, kh + c1 * D, bh + c1, cnt1, b, qv,
                                               sc + static_cast<int64_t>(pi) * b, sc + static_cast<int64_t>(pi + 1) * b,
                                               nullptr, nullptr);
                    } else {
                        scan_children<D, NVR>(kh + c0 * D, bh + c0, cnt0, b, qv, sc + static_cast<int64_t>(pi) * b);
                    }
                    continue;
                }
                if (pi + 1 < np) {
                    const int64_t c1 = static_cast<int64_t>(par[pi + 1]) * b;
                    const int cnt1 = static_cast<int>(min(static_cast<int64_t>(b), nl - c1));
                    for (int pl = 0; pl < R; ++pl)
                        scan_children<D, NVR>(kh + (c1 * R + pl) * D, bh + c1 * R + pl, cnt1, b, qv,
                                              sc + static_cast<int64_t>(pi + 1) * b, R * D, R, pl == 0);
                }
                for (int pl = 0; pl < R; ++pl)
                    scan_children<D, NVR>(kh + (c0 * R + pl) * D, bh + c0 * R + pl, cnt0, b, qv,
                                          sc + static_cast<int64_t>(pi) * b, R * D, R, pl == 0);
            }
            __syncwarp();
            const int nxt = nc <= kPRParents ? (cur == 0 ? 1 : 0) : (cur == 2 ? 3 : 2);
            auto node_of = [par, b](int i) { return static_cast<int32_t>(par[i / b] * b + i % b); };
            np = nc <= 64 ? top_p_small(sc, nc, a.p[l - 1], bufs[nxt], node_of)
                          : warp_top_p_binned(sc, nc, a.p[l - 1], bufs[nxt], node_of, sm.hist[w], sm.mem_key[w],
                                              sm.mem_mass[w]);
            __syncwarp();
            cur = nxt;
        }
        int32_t* out = a.sel + static_cast<int64_t>(x) * a.sel_cap;
        const int ncopy = min(np, a.sel_cap);
        for (int i = lane; i < ncopy; i += 32) out[i] = bufs[cur][i];
        if (lane == 0) {
            a.sel_count[x] = np;
            a.cand[x] = static_cast<int32_t>(scored);
            if (np > a.sel_cap) raise_status(ZHA_ERR_CAPACITY);
        }
        __syncwarp();
    }
}

// ======================================================================== plan
constexpr int kPairsPerRow = 8;     // partial slots per row, on average over a (sequence, KV head)
constexpr int kSBLog2Min = 2;       // superblocks of at least 4 blocks
constexpr int kSBOpts = 14;         // SB = 4 .. 32768 blocks
constexpr int kBitmapWords = 1024;  // union bitmap of one superblock (SB <= 32768)
constexpr int kPlanChunks = 32;     // CTAs per (sequence, KV head) in the per-row plan kernels
constexpr int kTileRows = 128;

struct PPlanArgs {
    const int32_t* sel;
    const int32_t* sel_count;
    const int32_t* n_tree;
    unsigned long long* totals;   // [slices][kSBOpts] pairs per superblock size
    int32_t* hdr;                 // [0] log2 SB, [1] superblocks per sequence (cap), [2] selected items
    int32_t* row_cnt;             // [slices * R] length of the row's valid (ascending, < n_1) list prefix
    int32_t* row_pairs;           // [slices * R]
    int32_t* row_off;             // [slices * R] global slot of the row's first partial
    int32_t* jcount;              // [slices][nJ_cap]
    int32_t* jcur;                // [slices][nJ_cap]
    int4* pairs;                  // [slices * R * kPairsPerRow] {row, first sel index, slot, 0}
    int4* items;                  // [item_cap] {slice, J, first pair, rows}
    int64_t nJ_cap, item_cap, n1_cap;
    int sel_cap, n_q, Hq, Hkv, G, B, R, slices;
};

// Row xr (slice-major: slice = xr / R, r = xr % R, query r / G, head r % G) ->
// its row in sel / sel_count / Q / O.
__device__ __forceinline__ int64_t prefill_sel_row(int64_t slice, int r, int Hkv, int Hq, int G, int n_q) {
    const int64_t s = slice / Hkv, h = slice % Hkv;
    return (s * n_q + r / G) * Hq + h * G + r % G;
}

// Pairs (row, superblock) for every superblock size: distinct superblocks of the
// row's blocks, plus superblock 0 for the sink when the row has not selected it.
__global__ void __launch_bounds__(256) prefill_count_kernel(PPlanArgs a) {
    __shared__ unsigned long long acc[kSBOpts];
    const int slice = blockIdx.x / kPlanChunks, chunk = blockIdx.x % kPlanChunks;
    if (threadIdx.x < kSBOpts) acc[threadIdx.x] = 0;
    __syncthreads();
    const int64_t n1 = a.n_tree[slice / a.Hkv] / a.B;
    unsigned long long c[kSBOpts];
#pragma unroll
    for (int o = 0; o < kSBOpts; ++o) c[o] = 0;
    if (n1 > 0) {
        for (int r = chunk * 256 + threadIdx.x; r < a.R; r += kPlanChunks * 256) {
            const int64_t row = prefill_sel_row(slice, r, a.Hkv, a.Hq, a.G, a.n_q);
            const int cnt = max(0, min(a.sel_count[row], a.sel_cap));
            const int32_t* list = a.sel + row * a.sel_cap;
            int prev[kSBOpts];
#pragma unroll
            for (int o = 0; o < kSBOpts; ++o) prev[o] = 0;   // superblock 0 always counts (sink)
#pragma unroll
            for (int o = 0; o < kSBOpts; ++o) c[o] += 1;
            int eff = 0, prevb = -1;
            for (int k = 0; k < cnt; ++k) {
                const int blk = list[k];
                if (blk <= prevb || blk >= n1) {   // not ascending or not a tree block: keep the prefix
                    raise_status(ZHA_ERR_INVALID_ARG);
                    break;
                }
                prevb = blk;
                ++eff;
#pragma unroll
                for (int o = 0; o < kSBOpts; ++o) {
                    const int J = blk >> (kSBLog2Min + o);
                    if (J != prev[o]) { c[o] += 1; prev[o] = J; }
                }
            }
            a.row_cnt[static_cast<int64_t>(slice) * a.R + r] = eff;
        }
    } else {
        for (int r = chunk * 256 + threadIdx.x; r < a.R; r += kPlanChunks * 256)
            a.row_cnt[static_cast<int64_t>(slice) * a.R + r] = 0;
    }
#pragma unroll
    for (int o = 0; o < kSBOpts; ++o) {
        const unsigned long long v = warp_sum_u64(c[o]);
        if ((threadIdx.x & 31) == 0 && v) atomicAdd(&acc[o], v);
    }
    __syncthreads();
    if (threadIdx.x < kSBOpts && acc[threadIdx.x]) atomicAdd(&a.totals[slice * kSBOpts + threadIdx.x], acc[threadIdx.x]);
}

// Picks SB and clears the per-superblock counters.  The pair totals it reads are
// zeroed on the stream before the count kernel of every plan.
__global__ void __launch_bounds__(1024) prefill_choose_kernel(PPlanArgs a) {
    __shared__ int s_log2;
    if (threadIdx.x == 0) {
        const unsigned long long cap = static_cast<unsigned long long>(a.R) * kPairsPerRow;
        int pick = kSBOpts - 1;
        for (int o = 0; o < kSBOpts; ++o) {
            bool ok = true;
            for (int s = 0; s < a.slices; ++s) ok = ok && a.totals[s * kSBOpts + o] <= cap;
            if (ok) { pick = o; break; }
        }
        s_log2 = kSBLog2Min + pick;
        a.hdr[0] = s_log2;
        a.hdr[1] = static_cast<int32_t>((a.n1_cap + (1ll << s_log2) - 1) >> s_log2);
        a.hdr[2] = 0;
    }
    __syncthreads();
    const int64_t nJ = (a.n1_cap + (1ll << s_log2) - 1) >> s_log2;
    for (int64_t i = threadIdx.x; i < static_cast<int64_t>(a.slices) * a.nJ_cap; i += blockDim.x) {
        if (i % a.nJ_cap < nJ) a.jcount[i] = 0;
    }
}

// Pairs per row at the chosen SB, and rows per superblock.
__global__ void __launch_bounds__(256) prefill_pairs_kernel(PPlanArgs a) {
    const int slice = blockIdx.x / kPlanChunks, chunk = blockIdx.x % kPlanChunks;
    const int lg = a.hdr[0];
    const int64_t n1 = a.n_tree[slice / a.Hkv] / a.B;
    int32_t* jc = a.jcount + static_cast<int64_t>(slice) * a.nJ_cap;
    for (int r = chunk * 256 + threadIdx.x; r < a.R; r += kPlanChunks * 256) {
        const int64_t row = prefill_sel_row(slice, r, a.Hkv, a.Hq, a.G, a.n_q);
        int c = 0;
        if (n1 > 0) {
            const int cnt = a.row_cnt[static_cast<int64_t>(slice) * a.R + r];
            const int32_t* list = a.sel + row * a.sel_cap;
            int prev = 0;
            c = 1;
            atomicAdd(&jc[0], 1);
            for (int k = 0; k < cnt; ++k) {
                const int J = list[k] >> lg;
                if (J != prev) { ++c; prev = J; atomicAdd(&jc[J], 1); }
            }
        }
        a.row_pairs[static_cast<int64_t>(slice) * a.R + r] = c;
    }
}

// Per (sequence, KV head): slots of each row's partials, first pair of each
// superblock, and the selected items (up to 128 rows of one superblock each).
__global__ void __launch_bounds__(1024) prefill_scan_kernel(PPlanArgs a) {
    __shared__ int scan[33];
    __shared__ int s_base;
    const int slice = blockIdx.x;
    const int64_t pair_base = static_cast<int64_t>(slice) * a.R * kPairsPerRow;
    const int lg = a.hdr[0];
    const int64_t nJ = (a.n1_cap + (1ll << lg) - 1) >> lg;
    // row slots: exclusive scan of row_pairs in row order
    int run = 0;
    for (int r0 = 0; r0 < a.R; r0 += 1024) {
        const int r = r0 + threadIdx.x;
        const int v = r < a.R ? a.row_pairs[static_cast<int64_t>(slice) * a.R + r] : 0;
        int tot;
        const int ex = block_exclusive_scan<32>(v, scan, &tot);
        if (r < a.R) a.row_off[static_cast<int64_t>(slice) * a.R + r] = static_cast<int32_t>(pair_base + run + ex);
        run += tot;
    }
    // superblocks: pair offsets (cursor for the scatter) and item counts
    int32_t* jc = a.jcount + static_cast<int64_t>(slice) * a.nJ_cap;
    int32_t* jr = a.jcur + static_cast<int64_t>(slice) * a.nJ_cap;
    int prun = 0, irun = 0;
    for (int64_t j0 = 0; j0 < nJ; j0 += 1024) {
        const int64_t J = j0 + threadIdx.x;
        const int cnt = J < nJ ? jc[J] : 0;
        const int nit = (cnt + kTileRows - 1) / kTileRows;
        int tp, ti;
        const int pex = block_exclusive_scan<32>(cnt, scan, &tp);
        const int iex = block_exclusive_scan<32>(nit, scan, &ti);
        if (J < nJ) {
            jr[J] = prun + pex;
            jc[J] = irun + iex;   // reused: first item of J inside the slice
        }
        prun += tp;
        irun += ti;
    }
    if (threadIdx.x == 0) s_base = atomicAdd(&a.hdr[2], irun);
    __syncthreads();
    const int base = s_base;
    for (int64_t J = threadIdx.x; J < nJ; J += 1024) {
        const int first = jc[J];
        const int next = J + 1 < nJ ? jc[J + 1] : irun;
        const int p0 = jr[J];
        const int cnt = (J + 1 < nJ ? jr[J + 1] : prun) - p0;
        for (int t = 0; t < next - first; ++t) {
            const int64_t it = static_cast<int64_t>(base) + first + t;
            if (it < a.item_cap)
                a.items[it] = make_int4(slice, static_cast<int>(J), static_cast<int>(pair_base + p0 + t * kTileRows),
                                        min(kTileRows, cnt - t * kTileRows));
        }
    }
}

// Writes every row's pairs into its superblock's bucket.
__global__ void __launch_bounds__(256) prefill_scatter_kernel(PPlanArgs a) {
    const int slice = blockIdx.x / kPlanChunks, chunk = blockIdx.x % kPlanChunks;
    const int lg = a.hdr[0];
    const int64_t n1 = a.n_tree[slice / a.Hkv] / a.B;
    if (n1 == 0) return;
    const int64_t pair_base = static_cast<int64_t>(slice) * a.R * kPairsPerRow;
    int32_t* jr = a.jcur + static_cast<int64_t>(slice) * a.nJ_cap;
    for (int r = chunk * 256 + threadIdx.x; r < a.R; r += kPlanChunks * 256) {
        const int64_t row = prefill_sel_row(slice, r, a.Hkv, a.Hq, a.G, a.n_q);
        const int cnt = a.row_cnt[static_cast<int64_t>(slice) * a.R + r];
        const int32_t* list = a.sel + row * a.sel_cap;
        int slot = a.row_off[static_cast<int64_t>(slice) * a.R + r];
        int pos = atomicAdd(&jr[0], 1);
        a.pairs[pair_base + pos] = make_int4(r, 0, slot++, 0);
        int prev = 0;
        for (int k = 0; k < cnt; ++k) {
            const int J = list[k] >> lg;
            if (J != prev) {
                prev = J;
                pos = atomicAdd(&jr[J], 1);
                a.pairs[pair_base + pos] = make_int4(r, k, slot++, 0);
            }
        }
    }
}

// ======================================================================== attention
struct PAttnArgs {
    const void* Q;            // bf16 [batch][n_q][Hq][D]
    float* O;                 // [batch][n_q][Hq][D] (dense mode)
    const int32_t* N;
    const int32_t* n_tree;
    const int32_t* sel;
    const int32_t* row_cnt;   // [slices * R] valid list length per row
    const int4* pairs;
    const int4* items;
    const int32_t* hdr;
    int32_t* ctr;             // [0] next item, [1] CTAs done; zero between calls
    float2* tail_ml;          // [slices * R]
    float* tail_o;            // [slices * R][D]
    float2* sel_ml;           // [slices * R * kPairsPerRow]
    float* sel_o;             // [slices * R * kPairsPerRow][D]
    int32_t* steps;           // [slices] 64-key blocks loaded (accounting)
    int64_t N_cap, item_cap;
    int sel_cap, n_q, Hq, Hkv, G, B, R, slices, tiles, dense;
    float qscale;             // softmax scale * log2(e)
};

struct PAttnCtl {
    uint64_t kv_full[2];      // TMA -> MMA: K and V of a block landed in buffer i
    uint64_t s_full[2];       // MMA -> softmax: S of the block in TMEM buffer i
    uint64_t p_full[2];       // softmax -> MMA: P of step g (buffer g & 1) written, O rescaled
    uint64_t o_done;          // MMA -> all: every MMA issued so far (through P V of the step) completed
    uint32_t tmem;
    int item;
    int abort;
    int pad;
    uint32_t bitmap[kBitmapWords];
};

constexpr int kPAThreads = 160;   // 4 softmax warps (one query row per thread) + 1 TMA/MMA warp
constexpr float kRescaleLog2 = 8.0f;   // lazy rescale: P stays below 2^8 between rescales

template <int D>
struct PAttnLayout {
    static constexpr int kH = D / 64;                          // 64-element column halves
    static constexpr uint32_t kQBytes = kH * kTileRows * 128;
    static constexpr uint32_t kKVBytes = kH * 64 * 128;        // one K or V block
    static constexpr uint32_t kPBytes = kTileRows * 128;       // 64 keys of bf16 per row
    static constexpr bool kPInK = kKVBytes >= kPBytes;         // P overwrites the consumed K block
    static constexpr uint32_t kOffK = kQBytes;
    static constexpr uint32_t kOffV = kOffK + 2 * kKVBytes;
    static constexpr uint32_t kOffP = kOffV + 2 * kKVBytes;    // two P buffers when P does not fit in K
    static constexpr uint32_t kOffCtl = kOffP + (kPInK ? 0 : 2 * kPBytes);
    static constexpr size_t kSmem = kOffCtl + sizeof(PAttnCtl) + 1024;   // + alignment slack
};

// Bounded wait; a timeout is recorded once and later waits of the CTA return at once.
__device__ __forceinline__ void pwait(uint64_t* bar, uint32_t parity, PAttnCtl* ctl) {
    if (*reinterpret_cast<volatile int*>(&ctl->abort)) return;
    if (!mbar_wait_bounded(bar, parity)) {
        ctl->abort = 1;
        raise_status(ZHA_ERR_TIMEOUT);
    }
}

__device__ __forceinline__ float fast_exp2(float x) {   // the SFU's 2^x (x = -inf gives +0)
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
        "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
        "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
        "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Iterates the key offsets of an item's blocks: the causal tail in order, or the
// set bits of the superblock bitmap in ascending order.
struct BlockCursor {
    bool tail;
    int64_t k0, jb0;
    int nwords, cw;
    uint32_t cbits;
    int k;
    __device__ __forceinline__ int64_t next(const uint32_t* bitmap) {
        if (tail) return k0 + static_cast<int64_t>(k++) * 64;
        while (cbits == 0u && cw + 1 < nwords) cbits = bitmap[++cw];
        const int bit = __ffs(cbits) - 1;
        cbits &= cbits - 1u;
        return (jb0 + cw * 32 + bit) * 64;
    }
};

template <int D>
__global__ void __launch_bounds__(kPAThreads, 2)
    attend_prefill_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          PAttnArgs a) {
    using Lay = PAttnLayout<D>;
    constexpr int H = Lay::kH;
    extern __shared__ __align__(1024) unsigned char pattn_smem[];
    const uint32_t raw_s = smem_addr(pattn_smem);
    unsigned char* base = pattn_smem + (((raw_s + 1023u) & ~1023u) - raw_s);
    unsigned char* sQ = base;
    unsigned char* sK = base + Lay::kOffK;
    unsigned char* sV = base + Lay::kOffV;
    PAttnCtl* ctl = reinterpret_cast<PAttnCtl*>(base + Lay::kOffCtl);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool softmax_role = warp < 4;

    if (warp == 0) {
        umma::tmem_alloc(&ctl->tmem, 256);
        umma::tmem_relinquish();
    }
    if (tid == 128) {
        mbar_init(&ctl->kv_full[0], 1);
        mbar_init(&ctl->kv_full[1], 1);
        mbar_init(&ctl->s_full[0], 1);
        mbar_init(&ctl->s_full[1], 1);
        mbar_init(&ctl->p_full[0], kTileRows);
        mbar_init(&ctl->p_full[1], kTileRows);
        mbar_init(&ctl->o_done, 1);
        fence_mbar_init();
        ctl->abort = 0;
        umma::prefetch_tensormap(&tmK);
        umma::prefetch_tensormap(&tmV);
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem;
    const uint32_t tO = tmem + 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr uint32_t kIdS = umma::idesc_bf16(128, 64, false);
    constexpr uint32_t kIdO = umma::idesc_bf16(128, D, true);
    uint32_t gstep = 0;        // blocks processed by this CTA so far (barrier phases follow it)
    const int n_tail = a.slices * a.tiles;
    const int64_t n_sel = a.dense ? 0 : (a.hdr[2] < a.item_cap ? a.hdr[2] : a.item_cap);
    const int n_total = n_tail + static_cast<int>(n_sel);
    auto p_buf = [&](uint32_t g) -> unsigned char* {
        return Lay::kPInK ? sK + (g & 1u) * Lay::kKVBytes : base + Lay::kOffP + (g & 1u) * Lay::kPBytes;
    };

    for (;;) {
        if (tid == 0) ctl->item = atomicAdd(&a.ctr[0], 1);
        __syncthreads();
        const int it = ctl->item;
        if (it >= n_total || *reinterpret_cast<volatile int*>(&ctl->abort)) break;
        // ---------------- the item and (softmax threads) this thread's row
        const bool tail = it < n_tail;
        int slice, r = 0, J = 0, selp = 0, nrows, row0 = 0;
        int64_t slot = 0;
        if (tail) {
            slice = it / a.tiles;
            row0 = (it % a.tiles) * kTileRows;
            nrows = min(kTileRows, a.R - row0);
            r = row0 + tid;
        } else {
            const int4 itm = a.items[it - n_tail];
            slice = itm.x;
            J = itm.y;
            nrows = itm.w;
            if (tid < nrows) {
                const int4 pr = a.pairs[itm.z + tid];
                r = pr.x;
                selp = pr.y;
                slot = pr.z;
            }
        }
        const int s = slice / a.Hkv;
        const int64_t N = a.N[s];
        const int64_t Ntree = a.dense ? 0 : a.n_tree[s];
        // the chunk's keys are in the cache and the tree covers exactly the keys before it
        const bool seq_ok = N >= a.n_q && N <= a.N_cap && (a.dense || Ntree == N - a.n_q);
        if (!seq_ok && tid == 0) raise_status(ZHA_ERR_INVALID_ARG);
        if (!seq_ok) nrows = 0;
        const bool row_ok = softmax_role && tid < nrows;
        const int64_t n1 = Ntree / a.B;
        const int64_t grow = prefill_sel_row(slice, r, a.Hkv, a.Hq, a.G, a.n_q);
        const int64_t t = N - a.n_q + r / a.G;
        const int32_t* list = a.sel + grow * a.sel_cap;
        const int lcnt = (!tail && row_ok) ? a.row_cnt[static_cast<int64_t>(slice) * a.R + r] : 0;
        BlockCursor cur{};
        cur.tail = tail;
        int nb = 0;
        if (tail) {
            cur.k0 = a.dense ? 0 : n1 * a.B;
            const int64_t tmax = N - a.n_q + (row0 + nrows - 1) / a.G;
            nb = nrows > 0 ? static_cast<int>((tmax + 1 - cur.k0 + 63) / 64) : 0;
        }
        // ---------------- Q rows -> swizzled K-major tile (softmax threads)
        if (softmax_role) {
            const uint16_t* qrow = static_cast<const uint16_t*>(a.Q) + grow * D;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const int half = c >> 3, cc = c & 7;
                unsigned char* dst = sQ + half * (kTileRows * 128) + tid * 128 + ((cc ^ (tid & 7)) << 4);
                umma::cp_async16(dst, row_ok ? static_cast<const void*>(qrow + c * 8) : a.Q, row_ok);
            }
        }
        // ---------------- selected item: union bitmap of the superblock's blocks
        if (!tail) {
            const int lg = a.hdr[0];
            const int64_t SB = 1ll << lg;
            cur.jb0 = static_cast<int64_t>(J) * SB;
            const int64_t jend = min(cur.jb0 + SB, n1);
            cur.nwords = static_cast<int>((jend - cur.jb0 + 31) / 32);
            for (int wi = tid; wi < cur.nwords; wi += kPAThreads) ctl->bitmap[wi] = 0u;
            __syncthreads();
            if (tid == 0 && J == 0) atomicOr(&ctl->bitmap[0], 1u);   // the sink's block
            if (row_ok) {
                for (int k = selp; k < lcnt && list[k] < jend; ++k) {   // ascending and >= jb0 by the plan
                    const int64_t bi = list[k] - cur.jb0;
                    atomicOr(&ctl->bitmap[bi >> 5], 1u << (bi & 31));
                }
            }
            __syncthreads();
            if (nrows > 0)
                for (int wi = 0; wi < cur.nwords; ++wi) nb += __popc(ctl->bitmap[wi]);
            cur.cbits = cur.nwords > 0 ? ctl->bitmap[0] : 0u;
        }
        if (softmax_role) umma::cp_async_wait_all();
        umma::fence_proxy_async_smem();
        __syncthreads();

        if (!softmax_role) {
            // ================= TMA + MMA issue (one lane)
            if (lane == 0 && nb > 0) {
                int64_t keys[2];
                auto issue = [&](int64_t key0, uint32_t buf) {
                    unsigned char* kd = sK + buf * Lay::kKVBytes;
                    unsigned char* vd = sV + buf * Lay::kKVBytes;
                    mbar_arrive_expect_tx(&ctl->kv_full[buf], 2 * Lay::kKVBytes);
#pragma unroll
                    for (int hh = 0; hh < H; ++hh) {
                        umma::tma_load_3d(kd + hh * 8192, &tmK, hh * 64, static_cast<int>(key0), slice, &ctl->kv_full[buf]);
                        umma::tma_load_3d(vd + hh * 8192, &tmV, hh * 64, static_cast<int>(key0), slice, &ctl->kv_full[buf]);
                    }
                };
                // waits for block (step g) in its buffer, zeroes V rows past the cache end
                auto land = [&](uint32_t g, int64_t key0) {
                    const uint32_t buf = g & 1u;
                    pwait(&ctl->kv_full[buf], (g >> 1) & 1u, ctl);
                    if (key0 + 64 > N) {
                        unsigned char* vb = sV + buf * Lay::kKVBytes;
                        const int valid = N > key0 ? static_cast<int>(N - key0) : 0;
                        for (int idx = 0; idx < (64 - valid) * H * 8; ++idx) {
                            const int rr = valid + idx / (H * 8), rest = idx % (H * 8);
                            *reinterpret_cast<uint4*>(vb + (rest >> 3) * 8192 + rr * 128 + ((rest & 7) << 4)) =
                                make_uint4(0u, 0u, 0u, 0u);
                        }
                        umma::fence_proxy_async_smem();
                    }
                };
                auto issue_s = [&](uint32_t g) {
                    const unsigned char* kb = sK + (g & 1u) * Lay::kKVBytes;
                    const uint32_t tS = tmem + (g & 1u) * 64;
                    umma::fence_after_sync();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = umma::desc_sw128(smem_addr(sQ + (kk >> 2) * (kTileRows * 128) + (kk & 3) * 32), 16, 1024);
                        const uint64_t bd = umma::desc_sw128(smem_addr(kb + (kk >> 2) * 8192 + (kk & 3) * 32), 16, 1024);
                        umma::mma_bf16(tS, ad, bd, kIdS, kk > 0 ? 1u : 0u);
                    }
                    umma::commit(&ctl->s_full[g & 1u]);
                };
                const uint32_t g0 = gstep;
                keys[0] = cur.next(ctl->bitmap);
                issue(keys[0], g0 & 1u);
                if (nb > 1) {
                    keys[1] = cur.next(ctl->bitmap);
                    issue(keys[1], (g0 + 1) & 1u);
                }
                land(g0, keys[0]);
                issue_s(g0);
                for (int k = 0; k < nb; ++k) {
                    const uint32_t g = g0 + k;
                    if (k + 1 < nb) {   // S of the next block overlaps this block's softmax
                        land(g + 1, keys[(k + 1) & 1]);
                        issue_s(g + 1);
                    }
                    pwait(&ctl->p_full[g & 1u], (g >> 1) & 1u, ctl);
                    umma::fence_after_sync();
                    const unsigned char* pb = p_buf(g);
                    const unsigned char* vb = sV + (g & 1u) * Lay::kKVBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma::desc_sw128(smem_addr(pb + kk * 32), 16, 1024);
                        const uint64_t bd = umma::desc_sw128(smem_addr(vb + kk * 2048), 8192, 1024);
                        umma::mma_bf16(tO, ad, bd, kIdO, (k > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma::commit(&ctl->o_done);
                    if (k + 2 < nb) {   // the block two ahead reuses this buffer once P V is done
                        pwait(&ctl->o_done, g & 1u, ctl);
                        keys[k & 1] = cur.next(ctl->bitmap);
                        issue(keys[k & 1], g & 1u);
                    }
                }
            }
        } else {
            // ================= masked online softmax, one query row per thread
            float m_run = -1e30f, l = 0.f;   // log2 domain; P = 2^(x - m_run) <= 2^8
            int64_t nsel_blk = (!tail && selp < lcnt) ? list[selp] : -1;
            for (int k = 0; k < nb; ++k) {
                const uint32_t g = gstep + k;
                const int64_t key0 = cur.next(ctl->bitmap);
                bool selected = false, sink_only = false;
                if (!tail && row_ok) {
                    const int64_t blk = key0 / 64;
                    selected = nsel_blk == blk;
                    if (selected) {
                        ++selp;
                        nsel_blk = selp < lcnt ? list[selp] : -1;
                    }
                    sink_only = !selected && blk == 0;
                }
                pwait(&ctl->s_full[g & 1u], (g >> 1) & 1u, ctl);
                umma::fence_after_sync();
                float sv[64];
                umma::tmem_ld32(tmem + (g & 1u) * 64 + lane_base, sv);
                umma::tmem_ld32(tmem + (g & 1u) * 64 + lane_base + 32, sv + 32);
                float mx = -INFINITY;
                if (tail) {
                    const int64_t lim = row_ok ? t - key0 : -1;   // keys key0 + c with c <= lim
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        sv[c] = c <= lim ? sv[c] * a.qscale : -INFINITY;
                        mx = fmaxf(mx, sv[c]);
                    }
                } else {
                    const int lim = selected ? 63 : (sink_only ? 0 : -1);
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        sv[c] = c <= lim ? sv[c] * a.qscale : -INFINITY;
                        mx = fmaxf(mx, sv[c]);
                    }
                }
                // lazy rescale: move the reference only when the row max outgrows it by 2^8
                bool resc = false;
                float alpha = 1.f;
                if (mx > m_run + kRescaleLog2) {
                    if (l > 0.f) {
                        resc = true;
                        alpha = fast_exp2(m_run - mx);
                        l *= alpha;
                    }
                    m_run = mx;
                }
                // P V of the previous block has completed (and with it every MMA issued
                // before it, S of this block included) before O is touched or P overwrites
                // this block's K.  (Relying on the S barrier alone for the overwrite raced:
                // a few rows came out wrong in some runs.)
                if (k > 0) pwait(&ctl->o_done, (g - 1) & 1u, ctl);
                if (__any_sync(0xffffffffu, resc) && k > 0) {
                    umma::fence_after_sync();
#pragma unroll
                    for (int q = 0; q < D / 32; ++q) {
                        float ov[32];
                        umma::tmem_ld32(tO + lane_base + q * 32, ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] *= alpha;
                        tmem_st32(tO + lane_base + q * 32, ov);
                    }
                    tmem_wait_st();
                }
                float ps = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const float p0 = fast_exp2(sv[c] - m_run), p1 = fast_exp2(sv[c + 1] - m_run);
                    ps += p0 + p1;
                    const __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
                    pk[c >> 1] = *reinterpret_cast<const uint32_t*>(&pb2);
                }
                l += ps;
                unsigned char* sP = p_buf(g);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    *reinterpret_cast<uint4*>(sP + tid * 128 + ((cc ^ (tid & 7)) << 4)) =
                        make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
                umma::fence_proxy_async_smem();
                umma::fence_before_sync();
                mbar_arrive(&ctl->p_full[g & 1u]);
            }
            // ---------------- this row's partial (or, dense, its output)
            if (nb > 0) {
                pwait(&ctl->o_done, (gstep + nb - 1) & 1u, ctl);
                umma::fence_after_sync();
                float* dst = nullptr;
                float scale = 1.f;
                if (row_ok) {
                    if (a.dense) {
                        dst = a.O + grow * D;
                        scale = 1.0f / l;
                    } else if (tail) {
                        const int64_t gx = static_cast<int64_t>(slice) * a.R + r;
                        a.tail_ml[gx] = make_float2(m_run, l);
                        dst = a.tail_o + gx * D;
                    } else {
                        a.sel_ml[slot] = make_float2(m_run, l);
                        dst = a.sel_o + slot * D;
                    }
                }
#pragma unroll
                for (int q = 0; q < D / 32; ++q) {
                    float ov[32];
                    umma::tmem_ld32(tO + lane_base + q * 32, ov);
                    if (dst) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(dst + q * 32 + e) =
                                make_float4(ov[e] * scale, ov[e + 1] * scale, ov[e + 2] * scale, ov[e + 3] * scale);
                    }
                }
                umma::fence_before_sync();
            }
        }
        if (tid == 0 && nb > 0) atomicAdd(&a.steps[slice], nb);
        gstep += nb;
        __syncthreads();
    }
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 256);
    }
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&a.ctr[1], 1) == static_cast<int>(gridDim.x) - 1) {
            a.ctr[0] = 0;
            a.ctr[1] = 0;
        }
    }
}

// ======================================================================== merge
struct PMergeArgs {
    float* O;
    const float2* tail_ml;
    const float* tail_o;
    const float2* sel_ml;
    const float* sel_o;
    const int32_t* row_pairs;
    const int32_t* row_off;
    int n_q, Hq, Hkv, G, R;
    int64_t rows;
};

// One warp per row: O = (sum_k 2^(m_k - M) o_k) / (sum_k 2^(m_k - M) l_k) over the
// row's tail partial and its superblock partials, in slot order.
template <int D>
__global__ void __launch_bounds__(256) merge_prefill_kernel(PMergeArgs a) {
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t xr = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
    if (xr >= a.rows) return;
    const int64_t slice = xr / a.R;
    const int r = static_cast<int>(xr % a.R);
    const int c = a.row_pairs[xr];
    const int64_t off = a.row_off[xr];
    const float2 mlt = a.tail_ml[xr];
    float M = mlt.x;
    for (int k = 0; k < c; ++k) M = fmaxf(M, a.sel_ml[off + k].x);
    float wt = exp2f(mlt.x - M);
    float lsum = mlt.y * wt;
    float acc[VF];
    load_n<float, VF>(a.tail_o + xr * D + lane * VF, acc);
#pragma unroll
    for (int e = 0; e < VF; ++e) acc[e] *= wt;
    for (int k = 0; k < c; ++k) {
        const float2 ml = a.sel_ml[off + k];
        const float w = exp2f(ml.x - M);
        lsum += ml.y * w;
        float x[VF];
        load_n<float, VF>(a.sel_o + (off + k) * D + lane * VF, x);
#pragma unroll
        for (int e = 0; e < VF; ++e) acc[e] = fmaf(x[e], w, acc[e]);
    }
    const float inv = 1.0f / lsum;
    float* dst = a.O + prefill_sel_row(slice, r, a.Hkv, a.Hq, a.G, a.n_q) * D + lane * VF;
#pragma unroll
    for (int e = 0; e < VF; ++e) dst[e] = acc[e] * inv;
}

}  // namespace zha
