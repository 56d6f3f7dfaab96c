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
//             scores are taken in ascending id order (ties to the lower id).  Up
//             to 64 candidates one warp sorts them; above that the whole block
//             bins them by score and ranks the crossing bin only (a single warp
//             doing the same takes ~18 ns per candidate: 12 us at 650).  Kept ids
//             stay ascending because children of ascending parents are ascending.
#pragma once

#include "zha_common.cuh"
#include "zha_topp.cuh"
#include "zha_plan.cuh"

namespace zha {

constexpr int kRouteThreads = 512;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kScoresSmem = 16384;   // candidate scores kept in shared memory up to this count
constexpr int kParentsSmem = 4096;   // per buffer; larger lists live in the workspace

struct RouteArgs {
    TreeDev tree;
    const void* Q;          // [batch][n_q][Hq][d]
    const int32_t* N;       // [batch]
    int32_t* sel;           // [batch][n_q][Hq][sel_cap]
    int32_t* sel_count;     // [batch][n_q][Hq]
    int32_t* cand;          // [batch][n_q][Hq] candidates scored over all levels (accounting)
    float* ws_scores;       // [batch*Hq][cand_cap]
    int32_t* ws_parents;    // [batch*Hq][2][par_cap]
    uint32_t* ws_ballot;    // [batch*Hq][2][kb_cap]
    int64_t cand_cap, par_cap, kb_cap, N_cap;
    PlanArgs plan;          // the gather plan, built here by the group's last CTA when fuse_plan
    uint32_t* grp_done;     // [batch*Hkv] query heads routed, zero between calls
    float2* pr_ml;          // value summaries (tree.vhat set): [batch*n_q*Hq] (max in log2 units, sum)
    float* pr_acc;          //   and [batch*n_q*Hq][d] of the nodes the cut dropped; else null
    int fuse_plan;
    int sel_cap, batch, Hq, Hkv, B, b, L_fixed, n_q;
    float scale;
    float p[kMaxLevels];
};

constexpr int kTieMax = 4096;   // crossing-bin members listed in shared memory (more: found by a scan)

struct RouteSmem {
    float scores[kScoresSmem];
    int32_t parents[2][kParentsSmem];
    unsigned long long bin_mass[1024];
    uint32_t keep_ballot[kScoresSmem / 32];
    int32_t keep_prefix[kScoresSmem / 32];
    int32_t tie_slot[kTieMax];
    float q[128];
    float pr_acc[128];                 // the dropped nodes' running value sum (value summaries)
    float pr_m, pr_l;                  //   its max (nats) and mass
    float pr_lw[kRouteWarps];          //   per-warp masses of one level
    int scan[kRouteWarps + 1];
    float redf[kRouteWarps];
    int redi[kRouteWarps];
    int plan_last;
    int tie_n, cut_bin;
    unsigned long long cut_above, cut_target;
};

// Top-p over sc[0..nc) (invalid slots hold -inf).  Writes the kept node ids,
// ascending, to out and returns their count.  node_of(i) maps a slot to its id.
constexpr int kBins = 1024;          // score bins of 1/32 nat below the level's max score
constexpr float kBinsPerNat = 32.0f;

__device__ __forceinline__ int score_bin(float s, float smax) {
    const float x = (smax - s) * kBinsPerNat;   // >= 0, weakly decreasing in s
    return x >= static_cast<float>(kBins - 1) ? kBins - 1 : static_cast<int>(x);
}

// Top-p cut over sc[0..nc) (invalid slots hold -inf): keeps the smallest prefix,
// in descending score order with ties to the lower slot (= lower node id), whose
// fixed-point mass reaches ceil(p * total).  Writes the kept node ids, ascending,
// to out; returns their count.  node_of(i) maps a slot to its node id.
//
// One pass bins the candidates by score (bins are monotone in the score, so the
// bin order is the sorted order up to the order inside a bin) and sums their
// masses per bin; one warp finds the bin where the cumulative mass crosses the
// target; only the candidates of that bin are ranked exactly (by score, then
// slot) against each other.  Candidate i is kept iff the mass of everything
// ordered before it is below the target.
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

// kball/kpre: ceil(nc/32) words each (shared memory, or the workspace for large nc).
template <typename NodeOf>
__device__ int top_p_select(const float* sc, int nc, float p, int32_t* out, RouteSmem& sm, uint32_t* kball,
                            int32_t* kpre, NodeOf node_of) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    // 1. max score; clear the bins
    float mx = -INFINITY;
    for (int i = tid; i < nc; i += kRouteThreads) mx = fmaxf(mx, sc[i]);
    mx = warp_max(mx);
    if (lane == 0) sm.redf[w] = mx;
    for (int k = tid; k < kBins; k += kRouteThreads) sm.bin_mass[k] = 0;
    if (tid == 0) { sm.tie_n = 0; sm.cut_above = 0; sm.cut_target = 0; }
    __syncthreads();
    mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kRouteWarps; ++i) mx = fmaxf(mx, sm.redf[i]);
    if (mx == -INFINITY) return 0;   // no candidates (uniform: every thread read the same partials)
    const bool keep_all = p >= 1.0f;
    int cbin = kBins;                 // keep_all: every valid candidate is "before the crossing bin"
    if (!keep_all) {
        // 2. mass per bin
        for (int i = tid; i < nc; i += kRouteThreads) {
            const float s = sc[i];
            if (s == -INFINITY) continue;
            atomicAdd(&sm.bin_mass[score_bin(s, mx)], score_mass(s, mx));
        }
        __syncthreads();
        // 3. one warp: total, target, the crossing bin and the mass of the bins before it.
        //    Lane j first sums bins [32j, 32j+32) (independent partial sums), then the
        //    crossing lane's 32 bins are scanned one per lane.
        if (w == 0) {
            const ulonglong2* bm = reinterpret_cast<const ulonglong2*>(sm.bin_mass + lane * 32);
            unsigned long long p0 = 0, p1 = 0, p2 = 0, p3 = 0;
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
                const ulonglong2 x = bm[k], y = bm[k + 1];
                p0 += x.x; p1 += x.y; p2 += y.x; p3 += y.y;
            }
            const unsigned long long ls = (p0 + p1) + (p2 + p3);
            unsigned long long incl = ls;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned long long tot = __shfl_sync(0xffffffffu, incl, 31);
            unsigned long long target =
                static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(tot)));
            if (target < 1) target = 1;
            if (target > tot) target = tot;
            const int J = __ffs(__ballot_sync(0xffffffffu, incl >= target)) - 1;
            const unsigned long long base = __shfl_sync(0xffffffffu, incl - ls, J);   // bins before lane J's
            const unsigned long long mb = sm.bin_mass[J * 32 + lane];
            unsigned long long run = mb;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += y;
            }
            const int k = __ffs(__ballot_sync(0xffffffffu, base + run >= target)) - 1;
            if (lane == k) {
                sm.cut_bin = J * 32 + k;
                sm.cut_above = base + run - mb;
                sm.cut_target = target;
            }
        }
        __syncthreads();
        cbin = sm.cut_bin;
        // 4. gather the crossing bin's candidates
        for (int i = tid; i < nc; i += kRouteThreads) {
            const float s = sc[i];
            if (s != -INFINITY && score_bin(s, mx) == cbin) {
                const int t = atomicAdd(&sm.tie_n, 1);
                if (t < kTieMax) sm.tie_slot[t] = i;
            }
        }
        __syncthreads();
    }
    const unsigned long long above = sm.cut_above, target = sm.cut_target;
    const int nt = sm.tie_n;
    // exact order inside the crossing bin: slot i of the bin is kept iff the mass of
    // the bin's members ordered before it (higher score, or equal score and lower
    // slot) plus the mass of the earlier bins stays below the target
    auto before_in_bin = [&](int i, float si) -> unsigned long long {
        unsigned long long bsum = 0;
        if (nt <= kTieMax) {
            for (int u = 0; u < nt; ++u) {
                const int j = sm.tie_slot[u];
                const float sj = sc[j];
                if (sj > si || (sj == si && j < i)) bsum += score_mass(sj, mx);
            }
        } else {   // more members than the list holds: scan every slot
            for (int j = 0; j < nc; ++j) {
                const float sj = sc[j];
                if (sj != -INFINITY && score_bin(sj, mx) == cbin && (sj > si || (sj == si && j < i)))
                    bsum += score_mass(sj, mx);
            }
        }
        return bsum;
    };
    auto kept = [&](int i) -> bool {
        const float s = sc[i];
        if (s == -INFINITY) return false;
        if (keep_all) return true;
        const int bn = score_bin(s, mx);
        return bn < cbin || (bn == cbin && above + before_in_bin(i, s) < target);
    };
    // 5. compaction in slot order: one ballot per 32-slot group (warp w takes groups
    //    w, w + 16, ...), an in-order prefix of the groups' counts by one warp, then writes
    const int ngrp = (nc + 31) / 32;
    for (int gi = w; gi < ngrp; gi += kRouteWarps) {
        const int i = gi * 32 + lane;
        const uint32_t bal = __ballot_sync(0xffffffffu, i < nc && kept(i));
        if (lane == 0) kball[gi] = bal;
    }
    __syncthreads();
    if (w == 0) {
        int run = 0;
        for (int gi = 0; gi < ngrp; gi += 32) {
            const int g2 = gi + lane;
            const int c = g2 < ngrp ? __popc(kball[g2]) : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (g2 < ngrp) kpre[g2] = run + incl - c;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) sm.redi[0] = run;
    }
    __syncthreads();
    const int total = sm.redi[0];
    for (int gi = w; gi < ngrp; gi += kRouteWarps) {
        const uint32_t bal = kball[gi];
        const int i = gi * 32 + lane;
        if ((bal >> lane) & 1u) out[kpre[gi] + __popc(bal & ((1u << lane) - 1u))] = node_of(i);
    }
    __syncthreads();
    return total;
}

// One warp scores the `cnt` (<= b <= NVR) children of one parent: rows of D fp32
// starting at kh, biases at bh.  NVR dot products are reduced together: after
// the halving steps lane holds row (lane >> (5 - log2 NVR)) of the block.
// With R planes per node, child r's plane p sits at kh[(r * R + p) * D]: the caller
// passes the plane's first row, rs = R * D and bs = R, and calls once per plane with
// first = (p == 0); later planes keep the max (the node's score is the max over planes).
template <int D, int NVR>
__device__ __forceinline__ void scan_children(const float* __restrict__ kh, const float* __restrict__ bh,
                                              int cnt, int b, const float* qv, float* __restrict__ out,
                                              int rs = D, int bs = 1, bool first = true) {
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
    if ((lane & ((1 << low) - 1)) == 0) {
        const int r = (lane >> low) & (NVR - 1);
        if (r < b) {
            const float t = r < cnt ? v[0] + bh[static_cast<int64_t>(r) * bs] : -INFINITY;
            out[r] = first ? t : fmaxf(out[r], t);
        }
    }
}

// scan_children for two parents at once: both blocks' loads are issued before either
// reduction, so a warp keeps twice the bytes in flight.
template <int D, int NVR>
__device__ __forceinline__ void scan_children2(const float* __restrict__ kh0, const float* __restrict__ bh0, int cnt0,
                                               const float* __restrict__ kh1, const float* __restrict__ bh1, int cnt1,
                                               int b, const float* qv, float* __restrict__ out0,
                                               float* __restrict__ out1, int rs = D, int bs = 1,
                                               bool first = true) {
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
    if ((lane & ((1 << low) - 1)) == 0) {
        const int r = (lane >> low) & (NVR - 1);
        if (r < b) {
            const float t0 = r < cnt0 ? v0[0] + bh0[static_cast<int64_t>(r) * bs] : -INFINITY;
            const float t1 = r < cnt1 ? v1[0] + bh1[static_cast<int64_t>(r) * bs] : -INFINITY;
            out0[r] = first ? t0 : fmaxf(out0[r], t0);
            out1[r] = first ? t1 : fmaxf(out1[r], t1);
        }
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
    // cross-warp sum: [warp][D] values through the (idle) block-cut bins, masses in pr_lw
    static_assert(kRouteWarps * 128 * sizeof(float) <= sizeof(RouteSmem::bin_mass), "scratch fits the bins");
    float* red = reinterpret_cast<float*>(sm.bin_mass);
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

// The top-down walk of one decode query (the body of route_decode_kernel).
template <typename T, int D, int NVR, bool MP, bool VS>
__device__ __forceinline__ void route_walk(const RouteArgs& a, RouteSmem& sm, int cta, int64_t row, int64_t slice,
                                           int64_t N, int64_t Ntree) {
    constexpr int VF = D / 32;   // fp32 summary elements per lane
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    (void)N;
    if (tid < D) sm.q[tid] = to_f32(static_cast<const T*>(a.Q)[row * D + tid]) * a.scale;
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
    int np = static_cast<int>((n[L - 1] + b - 1) / b);
    if (np > kParentsSmem) cur = 2;
    for (int i = tid; i < np; i += kRouteThreads) bufs[cur][i] = i;
    __syncthreads();

    int64_t scored = 0;
    for (int l = L; l >= 1; --l) {
        const int64_t nl = n[l - 1];
        const int nc = np * b;
        if (np > 0) {   // only the last possible parent can have fewer than b children
            const int64_t last_parent = (nl - 1) / b;
            scored += nc - (bufs[cur][np - 1] == last_parent ? b - (nl - last_parent * b) : 0);
        }
        float* sc = nc <= kScoresSmem ? sm.scores : ws_sc;
        const int32_t* par = bufs[cur];
        const int64_t ncap = a.tree.ncap[l - 1];
        const int R = MP ? a.tree.R : 1;
        const float* kh = a.tree.khat[l - 1] + slice * ncap * R * D;
        const float* bh = a.tree.bhat[l - 1] + slice * ncap * R;
        // ---- scan: one warp per kept parent, its b child rows of D fp32 (per plane, max over planes)
        for (int pi = w; pi < np; pi += 2 * kRouteWarps) {
            const int pj = pi + kRouteWarps;   // a second parent in the same round, if any
            const int64_t c0 = static_cast<int64_t>(par[pi]) * b;
            const int cnt0 = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
            if constexpr (!MP) {
                if (pj < np) {
                    const int64_t c1 = static_cast<int64_t>(par[pj]) * b;
                    const int cnt1 = static_cast<int>(min(static_cast<int64_t>(b), nl - c1));
                    scan_children2<D, NVR>(kh + c0 * D, bh + c0, cnt0, kh + c1 * D, bh + c1, cnt1, b, qv,
                                           sc + static_cast<int64_t>(pi) * b, sc + static_cast<int64_t>(pj) * b);
                } else {
                    scan_children<D, NVR>(kh + c0 * D, bh + c0, cnt0, b, qv, sc + static_cast<int64_t>(pi) * b);
                }
                continue;
            }
            if (pj < np) {
                const int64_t c1 = static_cast<int64_t>(par[pj]) * b;
                const int cnt1 = static_cast<int>(min(static_cast<int64_t>(b), nl - c1));
                for (int pl = 0; pl < R; ++pl)
                    scan_children<D, NVR>(kh + (c1 * R + pl) * D, bh + c1 * R + pl, cnt1, b, qv,
                                          sc + static_cast<int64_t>(pj) * b, R * D, R, pl == 0);
            }
            for (int pl = 0; pl < R; ++pl)
                scan_children<D, NVR>(kh + (c0 * R + pl) * D, bh + c0 * R + pl, cnt0, b, qv,
                                      sc + static_cast<int64_t>(pi) * b, R * D, R, pl == 0);
        }
        __syncthreads();
        // ---- top-p cut and compaction of the kept node ids
        const int np_par = np;
        const int nxt = nc <= kParentsSmem ? (cur == 0 ? 1 : 0) : (cur == 2 ? 3 : 2);
        auto node_of = [par, b](int i) { return static_cast<int32_t>(par[i / b] * b + i % b); };
        if (nc <= 64) {
            if (w == 0) {
                const int c = top_p_small(sc, nc, a.p[l - 1], bufs[nxt], node_of);
                if (lane == 0) sm.redi[0] = c;
            }
            __syncthreads();
            np = sm.redi[0];
        } else {
            const bool big = (nc + 31) / 32 > kScoresSmem / 32;
            np = top_p_select(sc, nc, a.p[l - 1], bufs[nxt], sm, big ? ws_kb : sm.keep_ballot,
                              big ? reinterpret_cast<int32_t*>(ws_kb) + a.kb_cap : sm.keep_prefix, node_of);
        }
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


// One CTA per (sequence, query head): the whole top-down walk of one decode query.
// NVR = b rounded up to a power of two (4, 8, 16 or 32).
// MP: nodes carry several reference-query planes (R > 1); R = 1 compiles the
// single-plane scan alone.  VS: the tree holds value summaries (R = 1): the nodes the
// cut drops are summed into a per-query partial.
template <typename T, int D, int NVR, bool MP, bool VS = false>
__global__ void __launch_bounds__(kRouteThreads, 1) route_decode_kernel(RouteArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    RouteSmem& sm = *reinterpret_cast<RouteSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int cta = blockIdx.x;
    const int s = cta / a.Hq, hq = cta % a.Hq;
    const int kv = hq / (a.Hq / a.Hkv);
    const int64_t slice = static_cast<int64_t>(s) * a.Hkv + kv;
    const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + hq;
    const int64_t N = a.N[s];
    const int64_t Ntree = a.tree.n_tree[s];
    const bool valid = !(N < 1 || N > a.N_cap || Ntree > N || Ntree < 0);
    if (!valid) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.sel_count[row] = 0; a.cand[row] = 0; }
    } else {
        route_walk<T, D, NVR, MP, VS>(a, sm, cta, row, slice, N, Ntree);
    }
    if (a.fuse_plan) {
        // the last of the group's G query-head CTAs builds the group's gather plan; the
        // count's release publishes this CTA's selection (ordered before it by the barrier),
        // its acquire makes the other heads' selections visible to the last CTA
        __syncthreads();
        if (tid == 0)
            sm.plan_last = atomic_add_acq_rel_gpu(&a.grp_done[slice], 1u) == static_cast<uint32_t>(a.Hq / a.Hkv - 1);
        __syncthreads();
        if (sm.plan_last) {
            plan_group(a.plan, static_cast<int>(slice), reinterpret_cast<uint32_t*>(sm.scores), sm.scan, N, Ntree);
            if (tid == 0) a.grp_done[slice] = 0u;
        }
    }
}

}  // namespace zha
