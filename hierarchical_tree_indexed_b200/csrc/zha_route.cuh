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
//             fixed-point integers (2^-40 units), so sums are order-free; a
//             radix select over the order-preserving 32-bit score keys finds the
//             cut score, equal scores are taken in ascending id order (ties to
//             the lower id), and a block scan compacts the kept ids, which stay
//             ascending because children of ascending parents are ascending.
#pragma once

#include "zha_common.cuh"

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
    int64_t cand_cap, par_cap, N_cap;
    int sel_cap, batch, Hq, Hkv, B, b, L_fixed, n_q;
    float scale;
    float p[kMaxLevels];
};

constexpr int kTieMax = 4096;   // crossing-bin members listed in shared memory (more: found by a scan)

struct RouteSmem {
    float scores[kScoresSmem];
    int32_t parents[2][kParentsSmem];
    unsigned long long bin_mass[1024];
    uint32_t bin_cnt[1024];
    int32_t tie_slot[kTieMax];
    float q[128];
    int scan[kRouteWarps + 1];
    float redf[kRouteWarps];
    int tie_n, cut_bin;
    unsigned long long cut_above, cut_target;
};

// Order-preserving key of a finite float (larger score -> larger key); -0 == +0.
__device__ __forceinline__ uint32_t score_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long score_mass(float s, float smax) {
    return __float2ull_rn(expf(s - smax) * 1099511627776.0f);   // 2^40
}

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
template <typename NodeOf>
__device__ int top_p_select(const float* sc, int nc, float p, int32_t* out, RouteSmem& sm, NodeOf node_of) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    // 1. max score; clear the bins
    float mx = -INFINITY;
    for (int i = tid; i < nc; i += kRouteThreads) mx = fmaxf(mx, sc[i]);
    mx = warp_max(mx);
    if (lane == 0) sm.redf[w] = mx;
    for (int k = tid; k < kBins; k += kRouteThreads) { sm.bin_mass[k] = 0; sm.bin_cnt[k] = 0; }
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
            const int bn = score_bin(s, mx);
            atomicAdd(&sm.bin_mass[bn], score_mass(s, mx));
            atomicAdd(&sm.bin_cnt[bn], 1u);
        }
        __syncthreads();
        // 3. one warp: total, target, the crossing bin and the mass of the bins before it
        if (w == 0) {
            unsigned long long ls = 0;
            for (int k = 0; k < kBins / 32; ++k) ls += sm.bin_mass[lane * (kBins / 32) + k];
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
            const uint32_t bal = __ballot_sync(0xffffffffu, incl >= target);
            const int J = __ffs(bal) - 1;            // first lane whose inclusive sum reaches the target
            if (lane == J) {
                unsigned long long run = incl - ls;  // mass of the bins of the lanes before J
                int c = lane * (kBins / 32);
                for (int k = 0; k < kBins / 32; ++k) {
                    const unsigned long long mk = sm.bin_mass[lane * (kBins / 32) + k];
                    if (run + mk >= target) { c = lane * (kBins / 32) + k; break; }
                    run += mk;
                }
                sm.cut_bin = c;
                sm.cut_above = run;
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
    // 5. compaction in slot order: thread t owns slots [t*per, (t+1)*per)
    const int per = (nc + kRouteThreads - 1) / kRouteThreads;
    const int i0 = min(nc, tid * per), i1 = min(nc, i0 + per);
    auto kept = [&](int i) -> bool {
        const float s = sc[i];
        if (s == -INFINITY) return false;
        if (keep_all) return true;
        const int bn = score_bin(s, mx);
        return bn < cbin || (bn == cbin && above + before_in_bin(i, s) < target);
    };
    int c = 0;
    for (int i = i0; i < i1; ++i) c += kept(i) ? 1 : 0;
    int total;
    int base = block_exclusive_scan<kRouteWarps>(c, sm.scan, &total);
    for (int i = i0; i < i1; ++i)
        if (kept(i)) out[base++] = node_of(i);
    __syncthreads();
    return total;
}

// One warp scores the `cnt` (<= b <= NVR) children of one parent: rows of D fp32
// starting at kh, biases at bh.  NVR dot products are reduced together: after
// the halving steps lane holds row (lane >> (5 - log2 NVR)) of the block.
template <int D, int NVR>
__device__ __forceinline__ void scan_children(const float* __restrict__ kh, const float* __restrict__ bh,
                                              int cnt, int b, const float* qv, float* __restrict__ out) {
    constexpr int VF = D / 32;
    const int lane = threadIdx.x & 31;
    float v[NVR];
#pragma unroll
    for (int r = 0; r < NVR; ++r) {
        float x[VF];
        if (r < cnt) {
            load_n<float, VF>(kh + static_cast<int64_t>(r) * D + lane * VF, x);
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
        if (r < b) out[r] = r < cnt ? v[0] + bh[r] : -INFINITY;
    }
}

// One CTA per (sequence, query head): the whole top-down walk of one decode query.
// NVR = b rounded up to a power of two (4, 8, 16 or 32).
template <typename T, int D, int NVR>
__global__ void __launch_bounds__(kRouteThreads, 1) route_decode_kernel(RouteArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    RouteSmem& sm = *reinterpret_cast<RouteSmem*>(smem_raw);
    constexpr int VF = D / 32;   // fp32 summary elements per lane
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int cta = blockIdx.x;
    const int s = cta / a.Hq, hq = cta % a.Hq;
    const int kv = hq / (a.Hq / a.Hkv);
    const int64_t slice = static_cast<int64_t>(s) * a.Hkv + kv;
    const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + hq;
    const int64_t N = a.N[s];
    const int64_t Ntree = a.tree.n_tree[s];
    if (N < 1 || N > a.N_cap || Ntree > N || Ntree < 0) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.sel_count[row] = 0; a.cand[row] = 0; }
        return;
    }
    if (tid < D) sm.q[tid] = to_f32(static_cast<const T*>(a.Q)[row * D + tid]) * a.scale;
    int64_t n[kMaxLevels];
    const int L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
    float qv[VF];
    __syncthreads();
#pragma unroll
    for (int e = 0; e < VF; ++e) qv[e] = sm.q[lane * VF + e];

    const int b = a.b;
    float* ws_sc = a.ws_scores + static_cast<int64_t>(cta) * a.cand_cap;
    int32_t* ws_par = a.ws_parents + static_cast<int64_t>(cta) * 2 * a.par_cap;
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
        const float* kh = a.tree.khat[l - 1] + slice * ncap * D;
        const float* bh = a.tree.bhat[l - 1] + slice * ncap;
        // ---- scan: one warp per kept parent, its b child rows of D fp32
        for (int pi = w; pi < np; pi += kRouteWarps) {
            const int64_t c0 = static_cast<int64_t>(par[pi]) * b;
            const int cnt = static_cast<int>(min(static_cast<int64_t>(b), nl - c0));
            scan_children<D, NVR>(kh + c0 * D, bh + c0, cnt, b, qv, sc + static_cast<int64_t>(pi) * b);
        }
        __syncthreads();
        // ---- top-p cut and compaction of the kept node ids
        const int nxt = nc <= kParentsSmem ? (cur == 0 ? 1 : 0) : (cur == 2 ? 3 : 2);
        auto node_of = [par, b](int i) { return static_cast<int32_t>(par[i / b] * b + i % b); };
        np = top_p_select(sc, nc, a.p[l - 1], bufs[nxt], sm, node_of);
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
}

}  // namespace zha
