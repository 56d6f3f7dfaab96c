// zha_route.cuh -- top-down top-p routing of decode queries.
//
// Page: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: at each level keep the smallest prefix of
// the candidates, ordered by score, whose normalised mass
//   sum_{i<=m} exp(s_i) / sum_{i<=n} exp(s_i)  reaches p  (the cut m_l(q)),
// then pass the kept nodes' children to the next level, down to the leaf
// blocks.  Scores are the tangent estimates s = scale * q.khat + bhat.
//
// One CTA walks the levels for one (sequence, query head), with no host round
// trip.  Per level:
//   scan   -- one warp per kept parent reads its b contiguous children (b*d fp32,
//             float4 per lane) and reduces b dot products at once with a
//             transpose-reduce over the warp;
//   top-p  -- exact and deterministic: masses exp(s - s_max) become 64-bit
//             fixed-point integers (2^-40 units), so sums are order-free; equal
//             scores are taken in ascending id order (ties to the lower id).  The
//             masses are binned by score below the level's max (which the scan
//             already found), one warp finds the bin where the cumulative mass
//             crosses p, and only that bin's members are ranked exactly (a dense
//             bin is split into sub-bins first).  Kept ids stay ascending
//             because children of ascending parents are ascending.
// The G query heads of one (sequence, KV head) run as one thread-block cluster:
// each head ORs its kept nodes into the shared memory of the cluster's CTA 0,
// which then builds the group's gather plan on chip.
#pragma once

#include "zha_common.cuh"
#include "zha_topp.cuh"
#include "zha_plan.cuh"

namespace zha {

constexpr int kRouteThreads = 512;
constexpr int kRouteWarps = kRouteThreads / 32;
// Shared memory is kept small on purpose: the scans' loads go through L1, which shares the SM's
// memory with it, and a smaller L1 holds fewer loads in flight.
constexpr int kScoresSmem = 8192;    // candidate scores kept in shared memory up to this count
constexpr int kParentsSmem = 2048;   // per buffer; larger lists live in the workspace

struct RouteArgs {
    TreeDev tree;
    const void* Q;          // [batch][n_q][Hq][d]
    const int32_t* N;       // [batch]
    int32_t* sel;           // [batch][n_q][Hq][sel_cap]
    int32_t* sel_count;     // [batch][n_q][Hq]
    int32_t* cand;          // [batch][n_q][Hq] candidates scored over all levels (accounting)
    float* ws_scores;       // [batch*Hq][cand_cap]
    int32_t* ws_parents;    // [batch*Hq][2][par_cap]
    uint32_t* ws_ballot;    // [batch*Hq][2][kb_cap] the cut's ballot words when they exceed shared memory
    int64_t cand_cap, par_cap, kb_cap, N_cap;
    PlanArgs plan;          // the gather plan, built here by the cluster's CTA 0 when fuse_plan
    int32_t* scanned;       // [batch*Hkv] distinct tree nodes the group's route read (fuse_plan)
    int lvl_off[kMaxLevels];// fuse_plan: word offset, in CTA 0's plan region, of level l's bitmap of
                            // kept nodes (index l-1, l >= 2); the G plan bitmaps start at word 0
    int region_words;       // words of the plan region (dynamic shared memory after RouteSmem)
    float2* pr_ml;          // value summaries (tree.vhat set): [batch*n_q*Hq] (max in log2 units, sum)
    float* pr_acc;          //   and [batch*n_q*Hq][d] of the nodes the cut dropped; else null
    int fuse_plan;          // the G CTAs of a group run as one cluster and build its plan
    int sel_cap, batch, Hq, Hkv, B, b, L_fixed, n_q;
    float scale;
    float p[kMaxLevels];
};

constexpr int kSpecMax = 256;   // the level below the top is scored with the top level when it has at most this many nodes
constexpr int kCutBins = 256;      // mass bins of 1/8 nat below the level's max score (a crossing bin
                                   // with too many members is split again into 256 sub-bins)
constexpr int kCutMembers = 256;   // crossing-bin members listed in shared memory and ranked pairwise
constexpr int kCutSplit = 64;      // a crossing bin with more members is split into sub-bins first

struct CutSmem {
    unsigned long long bins[kCutBins];     // zero between cuts
    uint32_t bw[2][kCutBins];              // a pass's masses as 32-bit words (low, high); zero between cuts
    unsigned long long mkey[kCutMembers];  // crossing-bin members: order key and mass
    unsigned long long mmass[kCutMembers];
    unsigned long long above, target;      // mass ordered before the crossing (sub-)bin; the target
    int nm, cbin, sbin;                    // members; crossing bin; crossing sub-bin (-1: not split)
    int cnt;                               // the kept count (small cuts)
};

// A level's scan offered to the other CTAs of the cluster (decode, the plan fused): the owner
// publishes where the jobs (kept parents) and their outputs are, then claims jobs from `claim`
// like its helpers.  Shared addresses are this CTA's; a helper maps them to the owner's.
// Only levels whose scores live in the workspace (more than kScoresSmem candidates) are
// offered: below that the claims' round trips cost more than the help saves (measured at 1M).
struct HelpSmem {
    uint32_t claim;            // (level << 24) | next job; jobs are claimed two at a time; 0: none
    uint32_t done;             // jobs of the offered level finished, helpers' included
    uint32_t walk_done;        // this CTA's walk is over: it offers nothing more
    int level, np, b;
    int64_t nl;                // nodes of the offered level
    const float* kh;           // the level's summaries and biases of this slice (global memory)
    const float* bh;
    float* sc_global;          // the scores, when they live in the workspace (the levels offered),
    uint32_t sc_smem;          //   else in this CTA's shared memory (helpers handle both)
    uint32_t par_smem;         // the kept parents in shared memory,
    const int32_t* par_global; //   or in the workspace
    uint32_t mx_smem;          // the level's max score slot (order-mapped int)
    uint32_t q_smem;           // the scaled query
};

struct RouteSmem {
    float scores[kScoresSmem];
    int32_t parents[2][kParentsSmem];
    float spec[kSpecMax + 32];         // scores of the level below the top, read with the top level
    CutSmem cut;
    uint32_t keep_ballot[kScoresSmem / 32];   // the cut's kept slots, a word per 32
    int32_t keep_prefix[kScoresSmem / 32];    // and the kept ids before each word
    float vred[kRouteWarps * 128];     // value summaries: per-warp value sums of one level
    float q[128];
    float pr_acc[128];                 // the dropped nodes' running value sum (value summaries)
    float pr_m, pr_l;                  //   its max (nats) and mass
    float pr_lw[kRouteWarps];          //   per-warp masses of one level
    int mxkey[2];                      // a level's max score (order-mapped), by level parity
    int scan[kRouteWarps + 1];
    float redf[kRouteWarps];
    int redi[kRouteWarps];
    HelpSmem help;                     // last: the buffers above keep their offsets
};

// Order-preserving map of a float (no NaN) to int, and back: the max of scores as an int max.
__device__ __forceinline__ int ord_key(float x) {
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float key_ord(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

// The same cut for nc <= 64, by warp 0 alone: the (score, slot) pairs are sorted by a
// bitonic network (descending score, ascending slot; two elements per lane), the
// fixed-point masses are prefix-summed in that order, and candidate e is kept iff the
// mass before it is below ceil(p * total).  The kept slots, ascending, go to out.
template <typename NodeOf>
__device__ int top_p_small(const float* sc, int nc, float p, int32_t* out, NodeOf node_of) {
    const int lane = threadIdx.x & 31;
    auto make = [&](int i) -> unsigned long long {
        const float s = i < nc ? sc[i] : -INFINITY;
        return s == -INFINITY ? 0ull
                              : (static_cast<unsigned long long>(score_key(s)) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
    };
    unsigned long long a = make(lane), b = make(lane + 32);   // elements lane and lane + 32
    for (int size = 2; size <= 64; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride == 32) {
                if (a < b) { const unsigned long long t = a; a = b; b = t; }   // size 64: descending
            } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    unsigned long long& x = h == 0 ? a : b;
                    const int e = lane + 32 * h;
                    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, stride);
                    const bool desc = (e & size) == 0;
                    const bool lower = (e & stride) == 0;
                    x = (lower == desc) ? (x > y ? x : y) : (x < y ? x : y);
                }
            }
        }
    }
    // sorted: element lane = a, element lane + 32 = b (descending); masses in that order
    const float smax = key_score(static_cast<uint32_t>(__shfl_sync(0xffffffffu, a, 0) >> 32));
    if (__shfl_sync(0xffffffffu, a, 0) == 0ull) return 0;   // no valid candidate
    const unsigned long long ma = a ? score_mass(key_score(static_cast<uint32_t>(a >> 32)), smax) : 0ull;
    const unsigned long long mb = b ? score_mass(key_score(static_cast<uint32_t>(b >> 32)), smax) : 0ull;
    unsigned long long ca = ma, cb = mb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long ya = __shfl_up_sync(0xffffffffu, ca, o);
        const unsigned long long yb = __shfl_up_sync(0xffffffffu, cb, o);
        if (lane >= o) { ca += ya; cb += yb; }
    }
    const unsigned long long half = __shfl_sync(0xffffffffu, ca, 31);
    cb += half;
    const unsigned long long tot = __shfl_sync(0xffffffffu, cb, 31);
    bool ka, kb;
    if (p >= 1.0f) {
        ka = a != 0ull;
        kb = b != 0ull;
    } else {
        unsigned long long target =
            static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(tot)));
        if (target < 1) target = 1;
        if (target > tot) target = tot;
        ka = a != 0ull && ca - ma < target;
        kb = b != 0ull && cb - mb < target;
    }
    // kept slots as a 64-bit set, then written in ascending slot order
    unsigned long long set = (ka ? 1ull << (0xffffffffu - static_cast<uint32_t>(a)) : 0ull) |
                             (kb ? 1ull << (0xffffffffu - static_cast<uint32_t>(b)) : 0ull);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) set |= __shfl_xor_sync(0xffffffffu, set, o);
    if ((set >> lane) & 1ull) out[__popcll(set & ((1ull << lane) - 1ull))] = node_of(lane);
    if ((set >> (lane + 32)) & 1ull) out[__popcll(set & ((1ull << (lane + 32)) - 1ull))] = node_of(lane + 32);
    return __popcll(set);
}

__device__ __forceinline__ int cut_bin(float s, float smax) {
    const float x = (smax - s) * 8.0f;   // >= 0, weakly decreasing in s
    return x >= static_cast<float>(kCutBins - 1) ? kCutBins - 1 : static_cast<int>(x);
}
// Sub-bin of s inside its bin `bin` (256 per bin; monotone in s within the bin).
__device__ __forceinline__ int cut_sub(float s, float smax, int bin) {
    const float f = ((smax - s) * 8.0f - static_cast<float>(bin)) * 256.0f;
    return f >= 255.0f ? 255 : static_cast<int>(f);
}
// Order of the candidates: by score, then the lower slot first.
__device__ __forceinline__ unsigned long long cut_key(float s, int i) {
    return (static_cast<unsigned long long>(score_key(s)) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
}

template <int NW>
__device__ __forceinline__ void cut_sync() {
    if constexpr (NW == 1) __syncwarp();
    else __syncthreads();
}

// Warp 0: the bin where base + the cumulative mass of bins[0..] reaches target (bins are 8
// rows of 32, lane j holding bins j + 32k, scanned as 8 independent warp scans); writes
// the bin to *bin_out and base + the mass of the bins before it to *above_out, and leaves
// the bins zero.  With target = 0 it first sets target = ceil(p * total), clamped to
// [1, total], and writes it to *target_io.
__device__ __forceinline__ void cut_locate(unsigned long long* bins, unsigned long long base, float p,
                                           unsigned long long* target_io, int* bin_out,
                                           unsigned long long* above_out) {
    const int lane = threadIdx.x & 31;
    unsigned long long v[8], in[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        v[k] = bins[lane + 32 * k];
        bins[lane + 32 * k] = 0ull;
        in[k] = v[k];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, in[k], o);
            if (lane >= o) in[k] += y;
        }
    unsigned long long rt[8], rp[8], tot = 0;   // row totals, exclusive prefix of the rows
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        rt[k] = __shfl_sync(0xffffffffu, in[k], 31);
        rp[k] = tot;
        tot += rt[k];
    }
    unsigned long long target = *target_io;
    if (target == 0ull) {
        target = static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(tot)));
        if (target < 1) target = 1;
        if (target > tot) target = tot;
    }
    int kc = 7;
#pragma unroll
    for (int k = 7; k >= 0; --k)
        if (base + rp[k] + rt[k] >= target) kc = k;
    unsigned long long inc = 0, val = 0, rpc = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (k == kc) { inc = in[k]; val = v[k]; rpc = rp[k]; }
    const uint32_t bal = __ballot_sync(0xffffffffu, base + rpc + inc >= target);
    const int lc = bal ? __ffs(bal) - 1 : 31;
    if (lane == lc) {
        *bin_out = 32 * kc + lc;
        *above_out = base + rpc + inc - val;
        *target_io = target;
    }
}

// Top-p cut over sc[0..nc) (invalid slots hold -inf) by the whole CTA: keeps the smallest
// prefix, in descending score order with ties to the lower slot (= lower node id), whose
// fixed-point mass reaches ceil(p * total); p >= 1 keeps every valid candidate.  mx is the
// max valid score (-inf: none).  Writes the kept node ids, ascending, to out and returns their
// count (in every thread).  cs.bins must be zero; they are left so.  kball, kpre: ceil(nc/32)
// words each (shared memory, or the workspace for large nc); scan: kRouteWarps + 1 ints.
//   1. every candidate's mass goes to its bin (1/8 nat below mx; masses below 2^-40 of the
//      max's are 0 and skipped);
//   2. warp 0 finds the bin where the cumulative mass reaches the target;
//   3. the candidates of earlier bins are kept (one ballot word per 32 slots) and the crossing
//      bin's members listed; when they are more than kCutSplit, their masses are binned again
//      into 256 sub-bins, the crossing sub-bin found, and its members listed instead;
//   4. member k is kept iff the mass of the members ordered before it, plus the mass ordered
//      before its (sub-)bin, is below the target (its bit joins the ballot words);
//   5. a scan of the ballot words' counts places every word's kept ids, in slot order.
// A pass adds each candidate's 64-bit mass to its bin as two 32-bit shared atomics (the low
// word, then the high word plus the low word's carry, only when not zero): thousands of
// candidates can share a bin, and contended 32-bit shared atomics are cheaper.  The words are
// gathered into cs.bins before the crossing bin is looked for.
// priv: when not null, kRouteWarps private pairs of word rows (shared memory otherwise idle),
// so that each warp's atomics go to its own words.
template <typename NodeOf>
__device__ int block_cut(const float* sc, int nc, float p, float mx, int32_t* out, CutSmem& cs, uint32_t* kball,
                         int32_t* kpre, int* scan, NodeOf node_of, unsigned long long* priv = nullptr) {
    constexpr int NT = kRouteThreads;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    if (mx == -INFINITY || nc <= 0) return 0;   // uniform
    if (nc <= 64) {   // one warp sorts them (top_p_small)
        if (w == 0) {
            const int c = top_p_small(sc, nc, p, out, node_of);
            if (lane == 0) cs.cnt = c;
        }
        __syncthreads();
        return cs.cnt;
    }
    const bool keep_all = p >= 1.0f;
    const int ngrp = (nc + 31) / 32;
    int cbin = kCutBins, sbin = -1;
    uint32_t* wlo = priv ? reinterpret_cast<uint32_t*>(priv) + w * 2 * kCutBins : cs.bw[0];   // this warp's words
    uint32_t* whi = wlo + kCutBins;
    auto add_mass = [&](int bn, unsigned long long m) {
        const uint32_t lo = static_cast<uint32_t>(m), hi = static_cast<uint32_t>(m >> 32);
        const uint32_t old = atomicAdd(&wlo[bn], lo);
        const uint32_t hc = hi + (old + lo < old ? 1u : 0u);   // the low word's carry
        if (hc) atomicAdd(&whi[bn], hc);
    };
    auto private_zero = [&]() {   // before a pass: this warp's words
        if (priv)
            for (int x = lane; x < 2 * kCutBins; x += 32) wlo[x] = 0u;
        __syncwarp();
    };
    auto gather = [&]() {   // after a pass and a barrier: the words into cs.bins (shared words left zero), a barrier
        for (int x = t; x < kCutBins; x += NT) {
            unsigned long long v = 0ull;
            if (priv) {
                for (int k = 0; k < kRouteWarps; ++k) {
                    const uint32_t* pw = reinterpret_cast<const uint32_t*>(priv) + k * 2 * kCutBins;
                    v += (static_cast<unsigned long long>(pw[kCutBins + x]) << 32) + pw[x];
                }
            } else {
                v = (static_cast<unsigned long long>(cs.bw[1][x]) << 32) + cs.bw[0][x];
                cs.bw[0][x] = 0u;
                cs.bw[1][x] = 0u;
            }
            cs.bins[x] = v;
        }
        __syncthreads();
    };
    if (!keep_all) {
        private_zero();
        for (int i = t; i < nc; i += NT) {
            const float s = sc[i];
            if (s == -INFINITY) continue;
            const unsigned long long m = score_mass(s, mx);
            if (m) add_mass(cut_bin(s, mx), m);
        }
        if (t == 0) { cs.nm = 0; cs.target = 0; cs.sbin = -1; }
        __syncthreads();
        gather();
        if (w == 0) cut_locate(cs.bins, 0ull, p, &cs.target, &cs.cbin, &cs.above);
        __syncthreads();
        cbin = cs.cbin;
    }
    // earlier bins as ballot words; the crossing bin's members listed
    for (int gi = w; gi < ngrp; gi += kRouteWarps) {
        const int i = gi * 32 + lane;
        const float s = i < nc ? sc[i] : -INFINITY;
        const int bn = s == -INFINITY ? kCutBins + 1 : (keep_all ? 0 : cut_bin(s, mx));
        const uint32_t bal = __ballot_sync(0xffffffffu, bn < cbin);
        if (lane == 0) kball[gi] = bal;
        if (bn == cbin) {
            const int k = atomicAdd(&cs.nm, 1);
            if (k < kCutMembers) {
                cs.mkey[k] = cut_key(s, i);
                cs.mmass[k] = score_mass(s, mx);
            }
        }
    }
    if (!keep_all) {
        __syncthreads();
        if (cs.nm > kCutSplit) {   // uniform: split the crossing bin (pairwise ranks grow as members^2)
            private_zero();
            for (int i = t; i < nc; i += NT) {
                const float s = sc[i];
                if (s != -INFINITY && cut_bin(s, mx) == cbin) {
                    const unsigned long long m = score_mass(s, mx);
                    if (m) add_mass(cut_sub(s, mx, cbin), m);
                }
            }
            __syncthreads();
            gather();
            if (t == 0) cs.nm = 0;
            if (w == 0) cut_locate(cs.bins, cs.above, p, &cs.target, &cs.sbin, &cs.above);
            __syncthreads();
            sbin = cs.sbin;
            for (int gi = w; gi < ngrp; gi += kRouteWarps) {   // earlier sub-bins join the ballots
                const int i = gi * 32 + lane;
                const float s = i < nc ? sc[i] : -INFINITY;
                const bool in_bin = s != -INFINITY && cut_bin(s, mx) == cbin;
                const int sb = in_bin ? cut_sub(s, mx, cbin) : 256;
                const uint32_t bal = __ballot_sync(0xffffffffu, sb < sbin);
                if (lane == 0 && bal) kball[gi] |= bal;
                if (in_bin && sb == sbin) {
                    const int k = atomicAdd(&cs.nm, 1);
                    if (k < kCutMembers) {
                        cs.mkey[k] = cut_key(s, i);
                        cs.mmass[k] = score_mass(s, mx);
                    }
                }
            }
            __syncthreads();
        }
        // the members: thread k ranks member k against the others
        const int nm = cs.nm;
        const unsigned long long above = cs.above, target = cs.target;
        if (nm <= kCutMembers) {
            for (int k = t; k < nm; k += NT) {
                const unsigned long long myk = cs.mkey[k];
                unsigned long long before = 0;
                for (int j = 0; j < nm; ++j)
                    if (cs.mkey[j] > myk) before += cs.mmass[j];
                if (above + before < target) {
                    const int i = static_cast<int>(0xffffffffu - static_cast<uint32_t>(myk));
                    atomicOr(&kball[i >> 5], 1u << (i & 31));
                }
            }
        } else {   // more members than the list holds even after the split: scan every slot
            for (int i = t; i < nc; i += NT) {
                const float s = sc[i];
                if (s == -INFINITY || cut_bin(s, mx) != cbin || (sbin >= 0 && cut_sub(s, mx, cbin) != sbin)) continue;
                const unsigned long long myk = cut_key(s, i);
                unsigned long long before = 0;
                for (int j = 0; j < nc; ++j) {
                    const float sj = sc[j];
                    if (sj != -INFINITY && cut_bin(sj, mx) == cbin && (sbin < 0 || cut_sub(sj, mx, cbin) == sbin) &&
                        cut_key(sj, j) > myk)
                        before += score_mass(sj, mx);
                }
                if (above + before < target) atomicOr(&kball[i >> 5], 1u << (i & 31));
            }
        }
    }
    __syncthreads();
    // ballot words -> positions (a thread per word, in rounds of NT words) -> ids in slot order
    int total = 0;
    for (int g0 = 0; g0 < ngrp; g0 += NT) {
        const int gi = g0 + t;
        int tot;
        const int x = block_exclusive_scan<kRouteWarps>(gi < ngrp ? __popc(kball[gi]) : 0, scan, &tot);
        if (gi < ngrp) kpre[gi] = total + x;
        total += tot;
    }
    __syncthreads();
    for (int gi = w; gi < ngrp; gi += kRouteWarps) {
        const uint32_t bal = kball[gi];
        if ((bal >> lane) & 1u) out[kpre[gi] + __popc(bal & ((1u << lane) - 1u))] = node_of(gi * 32 + lane);
    }
    return total;
}

// One warp scores the `cnt` (<= b <= NVR) children of one parent: rows of D fp32
// starting at kh, biases at bh.  NVR dot products are reduced together: after
// the halving steps lane holds row (lane >> (5 - log2 NVR)) of the block.
// With R planes per node, child r's plane p sits at kh[(r * R + p) * D]: the caller
// passes the plane's first row, rs = R * D and bs = R, and calls once per plane with
// first = (p == 0); later planes keep the max (the node's score is the max over planes).
// With mxk, the max of the scores written goes into *mxk (order-mapped, atomicMax): pass it
// on a candidate's last plane only.
template <int D, int NVR>
__device__ __forceinline__ void scan_children(const float* __restrict__ kh, const float* __restrict__ bh,
                                              int cnt, int b, const float* qv, float* __restrict__ out,
                                              int rs = D, int bs = 1, bool first = true, int* mxk = nullptr) {
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31;
    float v[NVR];
#pragma unroll
    for (int r = 0; r < NVR; ++r) {
        float x[VF];
        if (r < cnt) {
            load_n<float, VF>(kh + static_cast<int64_t>(r) * rs + lane * VF, x);
        } else {
#pragma unroll
            for (int e = 0; e < VF; ++e) x[e] = 0.f;
        }
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < VF; ++e) d = fmaf(qv[e], x[e], d);
        v[r] = d;
    }
    constexpr int H = NVR == 32 ? 5 : NVR == 16 ? 4 : NVR == 8 ? 3 : NVR == 4 ? 2 : 1;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        if (step < H) {
            const int half = NVR >> (step + 1);
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < NVR / 2; ++i) {
                if (i < half) {
                    const float send = upper ? v[i] : v[i + half];
                    const float keep = upper ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
    constexpr int low = 5 - H;
    int mk = ord_key(-INFINITY);
    if ((lane & ((1 << low) - 1)) == 0) {
        const int r = (lane >> low) & (NVR - 1);
        if (r < b) {
            const float t = r < cnt ? v[0] + bh[static_cast<int64_t>(r) * bs] : -INFINITY;
            const float val = first ? t : fmaxf(out[r], t);
            out[r] = val;
            mk = ord_key(val);
        }
    }
    if (mxk) {
        mk = __reduce_max_sync(0xffffffffu, mk);
        if (lane == 0) atomicMax(mxk, mk);
    }
}

// scan_children for two parents at once: both blocks' loads are issued before either
// reduction, so a warp keeps twice the bytes in flight.
template <int D, int NVR>
__device__ __forceinline__ void scan_children2(const float* __restrict__ kh0, const float* __restrict__ bh0, int cnt0,
                                               const float* __restrict__ kh1, const float* __restrict__ bh1, int cnt1,
                                               int b, const float* qv, float* __restrict__ out0,
                                               float* __restrict__ out1, int* mxk0, int* mxk1) {
    constexpr int rs = D, bs = 1;
    constexpr bool first = true;
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31;
    float x0[NVR][VF], x1[NVR][VF];
#pragma unroll
    for (int r = 0; r < NVR; ++r) {
        if (r < cnt0) load_n<float, VF>(kh0 + static_cast<int64_t>(r) * rs + lane * VF, x0[r]);
        else
#pragma unroll
            for (int e = 0; e < VF; ++e) x0[r][e] = 0.f;
        if (r < cnt1) load_n<float, VF>(kh1 + static_cast<int64_t>(r) * rs + lane * VF, x1[r]);
        else
#pragma unroll
            for (int e = 0; e < VF; ++e) x1[r][e] = 0.f;
    }
    float v0[NVR], v1[NVR];
#pragma unroll
    for (int r = 0; r < NVR; ++r) {
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int e = 0; e < VF; ++e) {
            d0 = fmaf(qv[e], x0[r][e], d0);
            d1 = fmaf(qv[e], x1[r][e], d1);
        }
        v0[r] = d0;
        v1[r] = d1;
    }
    constexpr int H = NVR == 32 ? 5 : NVR == 16 ? 4 : NVR == 8 ? 3 : NVR == 4 ? 2 : 1;
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        if (step < H) {
            const int half = NVR >> (step + 1);
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < NVR / 2; ++i) {
                if (i < half) {
                    const float s0 = upper ? v0[i] : v0[i + half], k0 = upper ? v0[i + half] : v0[i];
                    const float s1 = upper ? v1[i] : v1[i + half], k1 = upper ? v1[i + half] : v1[i];
                    v0[i] = k0 + __shfl_xor_sync(0xffffffffu, s0, o);
                    v1[i] = k1 + __shfl_xor_sync(0xffffffffu, s1, o);
                }
            }
        } else {
            v0[0] += __shfl_xor_sync(0xffffffffu, v0[0], o);
            v1[0] += __shfl_xor_sync(0xffffffffu, v1[0], o);
        }
    }
    constexpr int low = 5 - H;
    int mk0 = ord_key(-INFINITY), mk1 = ord_key(-INFINITY);
    if ((lane & ((1 << low) - 1)) == 0) {
        const int r = (lane >> low) & (NVR - 1);
        if (r < b) {
            const float t0 = r < cnt0 ? v0[0] + bh0[static_cast<int64_t>(r) * bs] : -INFINITY;
            const float t1 = r < cnt1 ? v1[0] + bh1[static_cast<int64_t>(r) * bs] : -INFINITY;
            out0[r] = first ? t0 : fmaxf(out0[r], t0);
            out1[r] = first ? t1 : fmaxf(out1[r], t1);
            mk0 = ord_key(t0);
            mk1 = ord_key(t1);
        }
    }
    if (mxk0) {
        mk0 = __reduce_max_sync(0xffffffffu, mk0);
        if (lane == 0) atomicMax(mxk0, mk0);
    }
    if (mxk1) {
        mk1 = __reduce_max_sync(0xffffffffu, mk1);
        if (lane == 0) atomicMax(mxk1, mk1);
    }
}

// Value summaries: the candidates of one level that the cut dropped (valid, not in the
// ascending kept list) join the running partial (sm.pr_m, sm.pr_l, sm.pr_acc) as pseudo-keys
// of log-mass s and value vhat.  Slots are parent-major (b per parent, as the scan wrote
// them); one warp per parent, lane r decides child r, the kept rows are skipped.
template <int D, int NVR>
__device__ void add_dropped(const float* sc, const int32_t* par, int np_par, int b, int64_t nl,
                            const int32_t* kept, int n_kept, const float* vh, RouteSmem& sm) {
    constexpr int VF = D / 32;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    auto is_kept = [&](int32_t node) {
        int lo = 0, hi = n_kept;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (kept[mid] < node) lo = mid + 1;
            else hi = mid;
        }
        return lo < n_kept && kept[lo] == node;
    };
    // the level's largest dropped score
    float mx = -INFINITY;
    for (int i = tid; i < np_par * b; i += kRouteThreads) {
        const float s = sc[i];
        if (s != -INFINITY && !is_kept(par[i / b] * b + i % b)) mx = fmaxf(mx, s);
    }
    mx = warp_max(mx);
    if (lane == 0) sm.redf[w] = mx;
    __syncthreads();
    mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kRouteWarps; ++i) mx = fmaxf(mx, sm.redf[i]);
    if (mx == -INFINITY) return;   // uniform: nothing dropped at this level
    const float m_old = sm.pr_m, m_new = fmaxf(m_old, mx);
    float acc[VF], lw = 0.f;
#pragma unroll
    for (int e = 0; e < VF; ++e) acc[e] = 0.f;
    for (int pi = w; pi < np_par; pi += kRouteWarps) {
        const int64_t c0 = static_cast<int64_t>(par[pi]) * b;
        const int cnt = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
        float wr = 0.f;
        if (lane < cnt) {
            const float s = sc[pi * b + lane];
            if (s != -INFINITY && !is_kept(static_cast<int32_t>(c0 + lane))) wr = expf(s - m_new);
        }
        lw += wr;
        const uint32_t mask = __ballot_sync(0xffffffffu, wr > 0.f);
        for (int r0 = 0; r0 < NVR; r0 += 4) {   // four rows' loads in flight at a time
            if (((mask >> r0) & 0xfu) == 0u) continue;
            float x[4][VF];
#pragma unroll
            for (int r = 0; r < 4; ++r)
                if ((mask >> (r0 + r)) & 1u) load_n<float, VF>(vh + (c0 + r0 + r) * D + lane * VF, x[r]);
#pragma unroll
            for (int r = 0; r < 4; ++r)
                if ((mask >> (r0 + r)) & 1u) {
                    const float e = __shfl_sync(0xffffffffu, wr, r0 + r);
#pragma unroll
                    for (int f = 0; f < VF; ++f) acc[f] = fmaf(e, x[r][f], acc[f]);
                }
        }
    }
    lw = warp_sum(lw);
    // cross-warp sum: [warp][D] values through vred, masses in pr_lw
    float* red = sm.vred;
#pragma unroll
    for (int f = 0; f < VF; ++f) red[w * D + lane * VF + f] = acc[f];
    if (lane == 0) sm.pr_lw[w] = lw;
    __syncthreads();
    const float alpha = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
    if (tid < D) {
        float t = 0.f;
#pragma unroll
        for (int ww = 0; ww < kRouteWarps; ++ww) t += red[ww * D + tid];
        sm.pr_acc[tid] = sm.pr_acc[tid] * alpha + t;
    }
    if (tid == 0) {
        float t = 0.f;
#pragma unroll
        for (int ww = 0; ww < kRouteWarps; ++ww) t += sm.pr_lw[ww];
        sm.pr_l = sm.pr_l * alpha + t;
        sm.pr_m = m_new;
    }
    __syncthreads();
}

// The scan of a level offered to the cluster (single plane): the descriptor is published
// (seqlock: level 0 while the fields change, the level after them, then the claim word with
// release order at cluster scope), the CTA's warps claim jobs two at a time like its helpers,
// and thread 0 waits (bounded) until every job is done, the helpers' included.  The caller's
// barrier follows.
template <int D, int NVR>
__device__ __forceinline__ void scan_offered(RouteSmem& sm, const float* kh, const float* bh, const int32_t* par,
                                          bool par_in_smem, int np, int b, int64_t nl, float* sc, int* mxk, int l,
                                          uint32_t head) {
    constexpr int VF = D / 32;
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) {
        HelpSmem& hs = sm.help;
        hs.level = 0;
        fence_acq_rel_cluster();
        hs.np = np;
        hs.b = b;
        hs.nl = nl;
        hs.kh = kh;
        hs.bh = bh;
        hs.sc_global = sc;
        hs.sc_smem = 0u;
        hs.par_smem = par_in_smem ? smem_addr(par) : 0u;
        hs.par_global = par_in_smem ? nullptr : par;
        hs.mx_smem = smem_addr(mxk);
        hs.q_smem = smem_addr(sm.q);
        hs.done = 0u;
        fence_acq_rel_cluster();
        hs.level = l;
        dsmem_st_release_u32(cluster_map(&hs.claim, head), static_cast<uint32_t>(l) << 24);
    }
    __syncthreads();
    float qv[VF];
#pragma unroll
    for (int e = 0; e < VF; ++e) qv[e] = sm.q[lane * VF + e];
    for (;;) {
        uint32_t jw = 0u;
        if (lane == 0) jw = atomicAdd(&sm.help.claim, 2u);
        jw = __shfl_sync(0xffffffffu, jw, 0);
        const int ji = static_cast<int>(jw & 0xffffffu);
        if ((jw >> 24) != static_cast<uint32_t>(l) || ji >= np) break;
        const int64_t c0 = static_cast<int64_t>(par[ji]) * b;
        const int cnt0 = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
        if (ji + 1 < np) {
            const int64_t c1 = static_cast<int64_t>(par[ji + 1]) * b;
            const int cnt1 = static_cast<int>(min(static_cast<int64_t>(b), nl - c1));
            scan_children2<D, NVR>(kh + c0 * D, bh + c0, cnt0, kh + c1 * D, bh + c1, cnt1, b, qv,
                                   sc + static_cast<int64_t>(ji) * b, sc + static_cast<int64_t>(ji + 1) * b, mxk, mxk);
        } else {
            scan_children<D, NVR>(kh + c0 * D, bh + c0, cnt0, b, qv, sc + static_cast<int64_t>(ji) * b, D, 1, true, mxk);
        }
        __syncwarp();
        if (lane == 0) atomicAdd(&sm.help.done, ji + 1 < np ? 2u : 1u);
    }
    if (tid == 0) {
        const uint32_t da = cluster_map(&sm.help.done, head);
        const uint64_t t0 = global_timer_ns();
        while (dsmem_ld_acquire_u32(da) < static_cast<uint32_t>(np))
            if (global_timer_ns() - t0 > kWaitLongNs) {
                raise_status(ZHA_ERR_TIMEOUT);
                break;
            }
    }
}

// The top-down walk of one decode query (the body of route_decode_kernel).  With
// `region` != 0 (fuse_plan) the kept nodes of every level are OR'd into the bitmaps of
// the cluster's CTA 0 (shared::cluster address of its plan region): level 1 into head
// `head`'s plan bitmap, level l >= 2 into the level's bitmap of kept nodes.  The walk
// then waits on the cluster barrier that CTA 0 arrived on after clearing the region,
// once, right after the top level's cut (before its first remote write).
template <typename T, int D, int NVR, bool MP, bool VS, bool HELP>
__device__ __forceinline__ void route_walk(const RouteArgs& a, RouteSmem& sm, int cta, int64_t row, int64_t slice,
                                           int64_t N, int64_t Ntree, uint32_t region, int head, float q_in) {
    constexpr int VF = D / 32;   // fp32 summary elements per lane
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    (void)N;
    if (tid < D) sm.q[tid] = q_in * a.scale;   // q_in: element tid of the query (loaded by the caller)
    if (tid < 2) sm.mxkey[tid] = ord_key(-INFINITY);
    for (int i = tid; i < kCutBins; i += kRouteThreads) {
        sm.cut.bins[i] = 0ull;
        sm.cut.bw[0][i] = 0u;
        sm.cut.bw[1][i] = 0u;
    }
    constexpr bool vsum = VS && !MP;   // value summaries (R = 1)
    if constexpr (vsum) {
        if (tid < D) sm.pr_acc[tid] = 0.f;
        if (tid == 0) { sm.pr_m = -INFINITY; sm.pr_l = 0.f; }
    }
    int64_t n[kMaxLevels];
    const int L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
    float qv[VF];
    __syncthreads();
#pragma unroll
    for (int e = 0; e < VF; ++e) qv[e] = sm.q[lane * VF + e];

    const int b = a.b;
    float* ws_sc = a.ws_scores + static_cast<int64_t>(cta) * a.cand_cap;
    int32_t* ws_par = a.ws_parents + static_cast<int64_t>(cta) * 2 * a.par_cap;
    uint32_t* ws_kb = a.ws_ballot + static_cast<int64_t>(cta) * 2 * a.kb_cap;
    int32_t* bufs[4] = {sm.parents[0], sm.parents[1], ws_par, ws_par + a.par_cap};
    int cur = 0;   // index into bufs

    // virtual parents of the top level: parent i has children [i*b, i*b+b) of level L
    int np = static_cast<int>((static_cast<uint32_t>(n[L - 1]) + b - 1) / static_cast<uint32_t>(b));
    if (np > kParentsSmem) cur = 2;
    for (int i = tid; i < np; i += kRouteThreads) bufs[cur][i] = i;
    // the level below the top, when small, is scored in the same pass as the top level (its
    // candidates are children of top nodes, known before the top level's cut): one round trip
    // to memory less; its scores wait in sm.spec for the cut to pick the kept parents' children
    const bool spec = L >= 2 && n[L - 2] <= kSpecMax;
    const int nspec = spec ? static_cast<int>(n[L - 1]) : 0;   // parents of the level below the top
    __syncthreads();

    int64_t scored = 0;
    for (int l = L; l >= 1; --l) {
        const int64_t nl = n[l - 1];
        const int nc = np * b;
        if (np > 0) {   // only the last possible parent can have fewer than b children
            const int64_t last_parent = static_cast<uint32_t>(nl - 1) / static_cast<uint32_t>(b);
            scored += nc - (bufs[cur][np - 1] == last_parent ? b - (nl - last_parent * b) : 0);
        }
        float* sc = nc <= kScoresSmem ? sm.scores : ws_sc;
        const int32_t* par = bufs[cur];
        const int64_t ncap = a.tree.ncap[l - 1];
        const int R = MP ? a.tree.R : 1;
        const float* kh = a.tree.khat[l - 1] + slice * ncap * R * D;
        const float* bh = a.tree.bhat[l - 1] + slice * ncap * R;
        int* mxk = &sm.mxkey[l & 1];   // this level's max score, found by the scan
        // the other slot is the next level's: its last reader, the cut one level up, is done
        if (tid == 0) sm.mxkey[(l + 1) & 1] = ord_key(-INFINITY);
        if (spec && l == L - 1) {
            // ---- the scores were read with the top level: the kept parents' children
            int mk = ord_key(-INFINITY);
            for (int i = tid; i < nc; i += kRouteThreads) {
                const int64_t c = static_cast<int64_t>(par[i / b]) * b + i % b;
                const float v = c < nl ? sm.spec[c] : -INFINITY;
                sc[i] = v;
                mk = max(mk, ord_key(v));
            }
            mk = __reduce_max_sync(0xffffffffu, mk);
            if (lane == 0) atomicMax(mxk, mk);
        } else {
            // ---- scan: one warp per parent (a job), its b child rows of D fp32 (per plane, max over
            //      planes); at the top level, jobs past the top's parents are the spec level's parents
            const int jobs = np + (l == L ? nspec : 0);
            const int64_t ncap_s = spec && l == L ? a.tree.ncap[L - 2] : 0;
            const float* kh_s = spec && l == L ? a.tree.khat[L - 2] + slice * ncap_s * R * D : nullptr;
            const float* bh_s = spec && l == L ? a.tree.bhat[L - 2] + slice * ncap_s * R : nullptr;
            // a job's max goes to this level's max, except the spec level's (its candidates are
            // only the kept top nodes' children, whose max the copy above takes)
            auto job = [&](int j, const float*& k0, const float*& b0, int& cnt, float*& out, int*& mx) {
                if (j < np) {
                    const int64_t c0 = static_cast<int64_t>(par[j]) * b;
                    cnt = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
                    k0 = kh + c0 * R * D;
                    b0 = bh + c0 * R;
                    out = sc + static_cast<int64_t>(j) * b;
                    mx = mxk;
                } else {
                    const int64_t c0 = static_cast<int64_t>(j - np) * b;
                    cnt = static_cast<int>(min(static_cast<int64_t>(b), n[L - 2] - c0));
                    k0 = kh_s + c0 * R * D;
                    b0 = bh_s + c0 * R;
                    out = sm.spec + c0;
                    mx = nullptr;
                }
            };
            auto two_jobs = [&](int ji, int jj) {   // jobs ji and jj (jj >= jobs: none)
                const float *k0, *b0, *k1 = nullptr, *b1 = nullptr;
                int cnt0, cnt1 = 0;
                float *o0, *o1 = nullptr;
                int *m0, *m1 = nullptr;
                job(ji, k0, b0, cnt0, o0, m0);
                if (jj < jobs) job(jj, k1, b1, cnt1, o1, m1);
                if constexpr (!MP) {
                    if (jj < jobs) scan_children2<D, NVR>(k0, b0, cnt0, k1, b1, cnt1, b, qv, o0, o1, m0, m1);
                    else scan_children<D, NVR>(k0, b0, cnt0, b, qv, o0, D, 1, true, m0);
                    return;
                }
                if (jj < jobs)
                    for (int pl = 0; pl < R; ++pl)
                        scan_children<D, NVR>(k1 + pl * D, b1 + pl, cnt1, b, qv, o1, R * D, R, pl == 0,
                                              pl == R - 1 ? m1 : nullptr);
                for (int pl = 0; pl < R; ++pl)
                    scan_children<D, NVR>(k0 + pl * D, b0 + pl, cnt0, b, qv, o0, R * D, R, pl == 0,
                                          pl == R - 1 ? m0 : nullptr);
            };
            // a large level below the top is offered to the cluster's CTAs whose walks are over
            bool offered = false;
            if constexpr (HELP && !MP && !vsum) {
                if (region != 0u && l < L && sc != sm.scores) {   // uniform
                    scan_offered<D, NVR>(sm, kh, bh, par, cur < 2, np, b, nl, sc, mxk, l, static_cast<uint32_t>(head));
                    offered = true;
                }
            }
            if (!offered) {
                for (int ji = w; ji < jobs; ji += 2 * kRouteWarps) two_jobs(ji, ji + kRouteWarps);   // two per round
            }
        }
        __syncthreads();
        // ---- top-p cut and compaction of the kept node ids
        const int np_par = np;
        const int nxt = nc <= kParentsSmem ? (cur == 0 ? 1 : 0) : (cur == 2 ? 3 : 2);
        auto node_of = [par, b](int i) { return static_cast<int32_t>(par[i / b] * b + i % b); };
        // the kept nodes into CTA 0's bitmaps: the level's kept set (for the count of distinct
        // nodes read), or at level 1 this head's selected blocks (the gather plan)
        auto publish = [&](int lv, const int32_t* kept, int cnt) {
            if (!region) return;
            const uint32_t bm = region + 4u * static_cast<uint32_t>(lv == 1 ? head * a.plan.words : a.lvl_off[lv - 1]);
            for (int i = tid; i < cnt; i += kRouteThreads) {
                const int32_t x = kept[i];
                dsmem_or(bm + 4u * static_cast<uint32_t>(x >> 5), 1u << (x & 31));
            }
        };
        if (!vsum && spec && l == L && nc <= 64 && cur < 2 && nxt < 2) {
            // ---- the top level and the level below it in one step of warp 0 (both small; the
            // level below was scored with the top): a block cut and the scores' copy less
            if (w == 0) {
                const int k = top_p_small(sc, nc, a.p[L - 1], bufs[nxt], node_of);
                __syncwarp();
                const int nc2 = k * b;
                int k2 = -1;
                if (nc2 <= 64) {
                    float* sc2 = sm.scores + 64;
                    const int32_t* kt = bufs[nxt];
                    for (int i = lane; i < nc2; i += 32) {
                        const int64_t c = static_cast<int64_t>(kt[i / b]) * b + i % b;
                        sc2[i] = c < n[L - 2] ? sm.spec[c] : -INFINITY;
                    }
                    __syncwarp();
                    auto node2 = [kt, b](int i) { return static_cast<int32_t>(kt[i / b] * b + i % b); };
                    k2 = top_p_small(sc2, nc2, a.p[L - 2], bufs[cur], node2);   // the top's parents are done
                }
                if (lane == 0) { sm.redi[0] = k; sm.redi[1] = k2; }
            }
            // the top level's max slot is the level two below's: clear it (its scan starts after
            // the barrier; nothing reads the top's max on this path)
            if (tid == 32) sm.mxkey[L & 1] = ord_key(-INFINITY);
            __syncthreads();
            const int k = sm.redi[0], k2 = sm.redi[1];
            if (region) cluster_wait();   // CTA 0 has cleared the region
            publish(L, bufs[nxt], k);
            if (k2 >= 0) {   // uniform
                publish(L - 1, bufs[cur], k2);
                const int64_t n2 = n[L - 2];
                const int64_t last2 = static_cast<uint32_t>(n2 - 1) / static_cast<uint32_t>(b);
                if (k > 0) scored += static_cast<int64_t>(k) * b - (bufs[nxt][k - 1] == last2 ? b - (n2 - last2 * b) : 0);
                np = k2;
                --l;   // the level below the top is done; bufs[cur] holds its kept nodes
                continue;
            }
            np = k;
            cur = nxt;
            continue;
        }
        {
            const bool big = (nc + 31) / 32 > kScoresSmem / 32;   // ballot words in the workspace
            // with the scores in the workspace, sm.scores holds the warps' private bins
            static_assert(kRouteWarps * 2 * kCutBins * sizeof(uint32_t) <= sizeof(float) * kScoresSmem,
                          "private bin words fit the score buffer");
            np = block_cut(sc, nc, a.p[l - 1], key_ord(*mxk), bufs[nxt], sm.cut, big ? ws_kb : sm.keep_ballot,
                           big ? reinterpret_cast<int32_t*>(ws_kb) + a.kb_cap : sm.keep_prefix, sm.scan, node_of,
                           sc != sm.scores ? reinterpret_cast<unsigned long long*>(sm.scores) : nullptr);
        }
        __syncthreads();
        if (region && l == L) cluster_wait();   // CTA 0 has cleared the region
        publish(l, bufs[nxt], np);
        if constexpr (vsum)
            add_dropped<D, NVR>(sc, par, np_par, b, nl, bufs[nxt], np, a.tree.vhat[l - 1] + slice * ncap * D, sm);
        cur = nxt;
    }
    // ---- level-1 selection -> sel
    const int32_t* fin = bufs[cur];
    int32_t* out = a.sel + row * a.sel_cap;
    const int ncopy = min(np, a.sel_cap);
    for (int i = tid; i < ncopy; i += kRouteThreads) out[i] = fin[i];
    if (tid == 0) {
        a.sel_count[row] = np;
        a.cand[row] = static_cast<int32_t>(scored);
        if (np > a.sel_cap) raise_status(ZHA_ERR_CAPACITY);
    }
    if constexpr (vsum) {   // the dropped nodes' partial, max in log2 units as the attention's partials
        if (tid < D) a.pr_acc[row * D + tid] = sm.pr_acc[tid];
        if (tid == 0) a.pr_ml[row] = make_float2(sm.pr_m * 1.4426950408889634f, sm.pr_l);
    }
}

// Distinct tree nodes the group's route read: every top node, the level below the top
// whole when it was read with the top (kSpecMax), and below that the children of the
// nodes any head kept one level up (the level bitmaps in the plan region).  One warp.
__device__ int64_t route_scanned(const RouteArgs& a, const uint32_t* region, int64_t Ntree) {
    const int lane = threadIdx.x & 31;
    int64_t n[kMaxLevels];
    const int L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
    const bool spec = L >= 2 && n[L - 2] <= kSpecMax;
    int64_t tot = n[L - 1] + (spec ? n[L - 2] : 0);
    for (int l = spec ? L - 1 : L; l >= 2; --l) {
        const uint32_t* bm = region + a.lvl_off[l - 1];
        const int64_t words = (n[l - 1] + 31) / 32, last = n[l - 1] - 1;
        int c = 0;
        for (int64_t i = lane; i < words; i += 32) c += __popc(bm[i]);
        c = __reduce_add_sync(0xffffffffu, static_cast<unsigned>(c));
        tot += static_cast<int64_t>(c) * a.b;
        if ((bm[last >> 5] >> (last & 31)) & 1u) tot -= a.b - (n[l - 2] - last * a.b);   // partial last parent
    }
    return tot;
}

// Writes the group's count of distinct nodes read (warp 1 of CTA 0, beside the plan's tail).
struct ScannedTail {
    const RouteArgs* a;
    const uint32_t* region;
    int64_t Ntree, slice;
    __device__ void operator()() const {
        const int64_t c = route_scanned(*a, region, Ntree);
        if ((threadIdx.x & 31) == 0) a->scanned[slice] = static_cast<int32_t>(c);
    }
};

// One CTA per (sequence, query head): the whole top-down walk of one decode query.
// NVR = b rounded up to a power of two (4, 8, 16 or 32).
// MP: nodes carry several reference-query planes (R > 1); R = 1 compiles the
// single-plane scan alone.  VS: the tree holds value summaries (R = 1): the nodes the
// cut drops are summed into a per-query partial.
// After its own walk, a CTA of the cluster scans jobs that the others offer (HelpSmem) until
// every other CTA's walk is over.  A warp claims two jobs at a time over DSMEM, reads the
// owner's descriptor and query the first time it meets an offer, scores the jobs into its own
// (now idle) score buffer, copies the scores where the owner keeps them, raises the owner's level
// max, and adds to its done count with release order.  Every wait is bounded.
template <int D, int NVR>
__device__ void route_help(RouteSmem& sm, uint32_t rank, uint32_t G) {
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (threadIdx.x == 0) dsmem_st_release_u32(cluster_map(&sm.help.walk_done, rank), 1u);
    float* scratch = sm.scores + w * 64;
    int c_rank = -1, c_level = -1, c_np = 0, c_b = 1;
    int64_t c_nl = 0;
    const float *c_kh = nullptr, *c_bh = nullptr;
    float* c_scg = nullptr;
    const int32_t* c_parg = nullptr;
    uint32_t c_scs = 0u, c_pars = 0u, c_mx = 0u, c_done = 0u;
    float qv[VF];
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        bool all_over = true, worked = false;
        for (uint32_t r = 0; r < G; ++r) {
            if (r == rank) continue;
            const uint32_t claim_r = cluster_map(&sm.help.claim, r);
            uint32_t wd = 0u, cw = 0u;
            if (lane == 0) {
                wd = dsmem_ld_acquire_u32(cluster_map(&sm.help.walk_done, r));
                cw = dsmem_ld_u32(claim_r);
            }
            wd = __shfl_sync(0xffffffffu, wd, 0);
            cw = __shfl_sync(0xffffffffu, cw, 0);
            if (!wd) all_over = false;
            if (cw == 0u) continue;   // nothing offered yet
            if (static_cast<int>(r) == c_rank && static_cast<int>(cw >> 24) == c_level &&
                static_cast<int>(cw & 0xffffffu) >= c_np)
                continue;   // that offer is taken up
            uint32_t jw = 0u;
            if (lane == 0) jw = dsmem_atom_add_u32(claim_r, 2u);
            jw = __shfl_sync(0xffffffffu, jw, 0);
            fence_acq_rel_cluster();   // the descriptor written before the claim word
            const int jl = static_cast<int>(jw >> 24), ji = static_cast<int>(jw & 0xffffffu);
            if (static_cast<int>(r) != c_rank || jl != c_level) {
                const uint32_t hb = cluster_map(&sm.help, r);
                auto fld = [&](const void* f) {
                    return hb + static_cast<uint32_t>(reinterpret_cast<const char*>(f) - reinterpret_cast<const char*>(&sm.help));
                };
                // seqlock read: the level before and after the fields must both be the claim's,
                // else the claim is a stale one of an offer the owner has closed
                int lv = 0;
                if (lane == 0) lv = static_cast<int>(dsmem_ld_u32(fld(&sm.help.level)));
                lv = __shfl_sync(0xffffffffu, lv, 0);
                if (lv != jl) continue;
                c_np = static_cast<int>(dsmem_ld_u32(fld(&sm.help.np)));
                c_b = static_cast<int>(dsmem_ld_u32(fld(&sm.help.b)));
                c_nl = static_cast<int64_t>(dsmem_ld_u64(fld(&sm.help.nl)));
                c_kh = reinterpret_cast<const float*>(dsmem_ld_u64(fld(&sm.help.kh)));
                c_bh = reinterpret_cast<const float*>(dsmem_ld_u64(fld(&sm.help.bh)));
                c_scg = reinterpret_cast<float*>(dsmem_ld_u64(fld(&sm.help.sc_global)));
                c_parg = reinterpret_cast<const int32_t*>(dsmem_ld_u64(fld(&sm.help.par_global)));
                const uint32_t scs = dsmem_ld_u32(fld(&sm.help.sc_smem)), pars = dsmem_ld_u32(fld(&sm.help.par_smem));
                c_scs = scs ? cluster_map_addr(scs, r) : 0u;
                c_pars = pars ? cluster_map_addr(pars, r) : 0u;
                c_mx = cluster_map_addr(dsmem_ld_u32(fld(&sm.help.mx_smem)), r);
                c_done = cluster_map(&sm.help.done, r);
                const uint32_t qa = cluster_map_addr(dsmem_ld_u32(fld(&sm.help.q_smem)), r);
#pragma unroll
                for (int e = 0; e < VF; ++e) qv[e] = dsmem_ld_f32(qa + 4u * static_cast<uint32_t>(lane * VF + e));
                fence_acq_rel_cluster();
                if (lane == 0) lv = static_cast<int>(dsmem_ld_u32(fld(&sm.help.level)));
                lv = __shfl_sync(0xffffffffu, lv, 0);
                if (lv != jl) {
                    c_rank = -1;
                    continue;
                }
                c_rank = static_cast<int>(r);
                c_level = jl;
            }
            if (ji >= c_np) continue;
            worked = true;
            const int nj = ji + 1 < c_np ? 2 : 1;
            auto par_of = [&](int j) {
                return c_pars ? static_cast<int32_t>(dsmem_ld_u32(c_pars + 4u * static_cast<uint32_t>(j))) : c_parg[j];
            };
            const int64_t p0 = par_of(ji), p1 = nj > 1 ? par_of(ji + 1) : 0;
            const int64_t c0 = p0 * c_b, c1 = p1 * c_b;
            const int cnt0 = static_cast<int>(min(static_cast<int64_t>(c_b), c_nl - c0));
            const int cnt1 = nj > 1 ? static_cast<int>(min(static_cast<int64_t>(c_b), c_nl - c1)) : 0;
            if (lane == 0) sm.redi[w] = ord_key(-INFINITY);
            __syncwarp();
            if (nj > 1)
                scan_children2<D, NVR>(c_kh + c0 * D, c_bh + c0, cnt0, c_kh + c1 * D, c_bh + c1, cnt1, c_b, qv, scratch,
                                       scratch + 32, &sm.redi[w], &sm.redi[w]);
            else
                scan_children<D, NVR>(c_kh + c0 * D, c_bh + c0, cnt0, c_b, qv, scratch, D, 1, true, &sm.redi[w]);
            __syncwarp();
            for (int x = lane; x < nj * c_b; x += 32) {   // the owner's slots ji b .. (ji + nj) b
                const float v = scratch[(x / c_b) * 32 + x % c_b];
                const int64_t dst = static_cast<int64_t>(ji) * c_b + x;
                if (c_scg) c_scg[dst] = v;
                else dsmem_st_f32(c_scs + 4u * static_cast<uint32_t>(dst), v);
            }
            __syncwarp();
            if (lane == 0) {
                dsmem_red_max_s32(c_mx, sm.redi[w]);
                dsmem_red_add_release_u32(c_done, static_cast<uint32_t>(nj));
            }
        }
        if (all_over) break;
        if (!worked) __nanosleep(256);   // polling: leave the owners' shared memory some quiet
        bool expired = false;
        if (lane == 0) expired = !worked && global_timer_ns() - t0 > kWaitLongNs;
        if (__shfl_sync(0xffffffffu, expired, 0)) {
            if (lane == 0) raise_status(ZHA_ERR_TIMEOUT);
            break;
        }
    }
}

// fuse_plan: launched as clusters of G CTAs, the G query heads of one (sequence, KV
// head) (cluster rank = head).  CTA 0 clears its plan region, the heads OR their kept
// nodes into it (DSMEM), and after a cluster barrier CTA 0 builds the group's gather
// plan from its own shared memory.
// HELP: the cluster's CTAs help each other scan levels too large for shared memory (chosen by
// the host where the launch leaves SMs idle; the code is not compiled into the other variants).
template <typename T, int D, int NVR, bool MP, bool VS = false, bool HELP = false>
__global__ void __launch_bounds__(kRouteThreads, 1) route_decode_kernel(RouteArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    RouteSmem& sm = *reinterpret_cast<RouteSmem*>(smem_raw);
    uint32_t* region = reinterpret_cast<uint32_t*>(smem_raw + sizeof(RouteSmem));
    const int tid = threadIdx.x;
    const int cta = blockIdx.x;
    const int s = cta / a.Hq, hq = cta % a.Hq;
    const int G = a.Hq / a.Hkv;
    const int kv = hq / G;
    const int64_t slice = static_cast<int64_t>(s) * a.Hkv + kv;
    const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + hq;
    const bool fused = a.fuse_plan != 0;
    // the query, the key count and the tree count in one round trip to memory
    const float q_in = tid < D ? to_f32(static_cast<const T*>(a.Q)[row * D + tid]) : 0.f;
    const uint32_t rank = fused ? cluster_rank() : 0u;
    if (fused) {
        if (rank == 0)
            for (int i = tid; i < a.region_words; i += kRouteThreads) region[i] = 0u;
        if constexpr (HELP)
            if (tid == 0) {
                sm.help.claim = 0u;
                sm.help.done = 0u;
                sm.help.walk_done = 0u;
                sm.help.level = 0;
            }
        cluster_arrive();   // waited on by the walk before its first remote write (or help)
    }
    const int64_t N = a.N[s];
    const int64_t Ntree = a.tree.n_tree[s];
    const bool valid = !(N < 1 || N > a.N_cap || Ntree > N || Ntree < 0);   // uniform over the cluster
    if (!valid) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.sel_count[row] = 0; a.cand[row] = 0; }
        if (fused) cluster_wait();
    } else {
        route_walk<T, D, NVR, MP, VS, HELP>(a, sm, cta, row, slice, N, Ntree, fused ? cluster_map(region, 0) : 0u,
                                            static_cast<int>(rank), q_in);
        if constexpr (HELP && !MP && !VS)
            if (fused && G > 1) route_help<D, NVR>(sm, rank, static_cast<uint32_t>(G));
    }
    if (fused) {
        // every head's kept nodes are in CTA 0's region; the other CTAs are done with it
        cluster_arrive();
        cluster_wait();
        if (rank == 0) {
            if (valid) {
                plan_emit(a.plan, static_cast<int>(slice), region, sm.scan, N, Ntree,
                          ScannedTail{&a, region, Ntree, slice});
            } else if (tid == 0) {
                a.plan.n_items[slice] = 0;
                a.plan.rows[slice] = 0;
                a.scanned[slice] = 0;
            }
        }
    }
}

}  // namespace zha
