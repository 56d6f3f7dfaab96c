// zha_topp.cuh -- the top-p cut of one level's candidates, the rule both routers
// apply, and its warp-level forms.
//
// Page: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: keep the smallest prefix of the candidates,
// in descending score order, whose normalised mass reaches p.  Masses are
// exp(s - s_max) as 64-bit fixed-point integers (2^-40 units), so sums do not
// depend on their order; ties go to the lower candidate id.
#pragma once

#include "zha_common.cuh"

namespace zha {

constexpr int kWarpCutBins = 256;      // per-warp mass histogram of the binned cut (1/32 nat bins)
constexpr int kWarpCutMembers = 64;    // crossing-bin members ranked exactly in shared memory

// Order-preserving key of a finite float (larger score -> larger key); -0 == +0.
__device__ __forceinline__ uint32_t score_key(float s) {
    const uint32_t u = __float_as_uint(s + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ unsigned long long score_mass(float s, float smax) {
    return __float2ull_rn(expf(s - smax) * 1099511627776.0f);   // 2^40
}

__device__ __forceinline__ float key_score(uint32_t k) {   // inverse of score_key
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
// Top-p cut of one warp over sc[0..nc): the same kept set as top_p_select (the
// smallest prefix in descending score order, ties to the lower slot, whose
// fixed-point mass reaches ceil(p * total)).  The cut key K is the largest score
// key whose upper mass M(>= K) still reaches the target, found by bisection;
// every candidate above K is kept, and candidates equal to K are kept in slot
// order while the mass before them stays below target - M(> K).  Writes the kept
// ids ascending to out and returns their count.  (The tie pass walks the tied
// lanes with a ballot: an optimised build of a 64-bit shuffle-scan form of it
// dropped the crossing candidate, while the same source was exact unoptimised.)
template <typename NodeOf>
__device__ int warp_top_p(const float* sc, int nc, float p, int32_t* out, NodeOf node_of) {
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int i = lane; i < nc; i += 32) mx = fmaxf(mx, sc[i]);
    mx = warp_max(mx);
    if (mx == -INFINITY) return 0;
    const bool keep_all = p >= 1.0f;
    unsigned long long tot = 0;
    uint32_t klo = 0xffffffffu;
    for (int i = lane; i < nc; i += 32) {
        const float s = sc[i];
        if (s != -INFINITY) {
            tot += score_mass(s, mx);
            klo = min(klo, score_key(s));
        }
    }
    tot = warp_sum_u64(tot);
    klo = warp_min_u32(klo);
    unsigned long long target =
        static_cast<unsigned long long>(ceil(static_cast<double>(p) * static_cast<double>(tot)));
    if (target < 1) target = 1;
    if (target > tot) target = tot;
    uint32_t lo = klo, hi = keep_all ? klo : score_key(mx);   // M(>= lo) = tot >= target
    while (lo < hi) {
        const uint32_t mid = lo + (hi - lo + 1) / 2;
        unsigned long long m = 0;
        for (int i = lane; i < nc; i += 32) {
            const float s = sc[i];
            if (s != -INFINITY && score_key(s) >= mid) m += score_mass(s, mx);
        }
        m = warp_sum_u64(m);
        if (m >= target) lo = mid;
        else hi = mid - 1;
    }
    const uint32_t K = lo;
    unsigned long long above = 0;
    for (int i = lane; i < nc; i += 32) {
        const float s = sc[i];
        if (s != -INFINITY && score_key(s) > K) above += score_mass(s, mx);
    }
    const unsigned long long need = target - warp_sum_u64(above);
    int cnt = 0;
    unsigned long long carry = 0;
    for (int base = 0; base < nc; base += 32) {
        const int i = base + lane;
        const float s = i < nc ? sc[i] : -INFINITY;
        const bool valid = s != -INFINITY;
        const uint32_t k = valid ? score_key(s) : 0u;
        const bool tie = !keep_all && valid && k == K;
        const unsigned long long mm = tie ? score_mass(s, mx) : 0ull;
        // candidates equal to the cut key, in slot order: kept while the tie mass
        // ahead of them is below `need` (a ballot walk: ties are few)
        uint32_t tb = __ballot_sync(0xffffffffu, tie);
        bool keep_tie = false;
        while (tb) {
            const int j = __ffs(tb) - 1;
            tb &= tb - 1u;
            const unsigned long long mj = __shfl_sync(0xffffffffu, mm, j);
            if (lane == j) keep_tie = carry < need;
            carry += mj;
        }
        const bool keep = valid && (keep_all || k > K || keep_tie);
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) out[cnt + __popc(bal & ((1u << lane) - 1u))] = node_of(i);
        cnt += __popc(bal);
    }
    return cnt;
}

// The same cut as warp_top_p, found with a histogram: one pass sums the fixed-point
// masses into bins of 1/32 nat below the max score (bins are monotone in the score,
// so bin order is the sorted order up to the order inside a bin); a warp scan finds
// the bin where the cumulative mass reaches ceil(p * total); only that bin's members
// are ranked exactly (score, then slot), by comparing each against the others.
// Falls back to warp_top_p when the crossing bin holds more than kWarpCutMembers.
// NB bins of 1/32 nat (a multiple of 32); the last bin takes everything further below the
// max, and its mass is summed in registers (it is the bin most candidates share).  The other
// bins take each 64-bit mass as two 32-bit shared atomics, the low word and then the high word
// plus the low word's carry when not zero (hist read as 2 NB words: low words first): 64-bit
// shared-memory atomics of a warp to one address serialise far more (measured ~27x).
template <int NB = kWarpCutBins, typename NodeOf>
__device__ int warp_top_p_binned(const float* sc, int nc, float p, int32_t* out, NodeOf node_of,
                                 unsigned long long* hist, unsigned long long* mkey,
                                 unsigned long long* mmass) {
    static_assert(NB % 32 == 0, "bins per lane");
    const int lane = threadIdx.x & 31;
    if (p >= 1.0f) return warp_top_p(sc, nc, p, out, node_of);
    float mx = -INFINITY;
    for (int i = lane; i < nc; i += 32) mx = fmaxf(mx, sc[i]);
    mx = warp_max(mx);
    if (mx == -INFINITY) return 0;
    auto bin_of = [mx](float s) -> int {
        const float x = (mx - s) * 32.0f;
        return x >= static_cast<float>(NB - 1) ? NB - 1 : static_cast<int>(x);
    };
#pragma unroll
    for (int k = 0; k < NB / 32; ++k) hist[lane + 32 * k] = 0ull;   // both word rows
    __syncwarp();
    uint32_t* hw = reinterpret_cast<uint32_t*>(hist);
    unsigned long long far = 0;
    for (int i = lane; i < nc; i += 32) {
        const float s = sc[i];
        if (s == -INFINITY) continue;
        const int bn = bin_of(s);
        const unsigned long long m = score_mass(s, mx);
        if (bn == NB - 1) {
            far += m;
        } else {
            const uint32_t lo = static_cast<uint32_t>(m), hi = static_cast<uint32_t>(m >> 32);
            const uint32_t old = atomicAdd(&hw[bn], lo);
            const uint32_t hc = hi + (old + lo < old ? 1u : 0u);
            if (hc) atomicAdd(&hw[NB + bn], hc);
        }
    }
    far = warp_sum_u64(far);
    __syncwarp();
    if (lane == 0) {
        hw[NB - 1] = static_cast<uint32_t>(far);
        hw[2 * NB - 1] = static_cast<uint32_t>(far >> 32);
    }
    __syncwarp();
    // lane j owns bins [j NB/32, (j+1) NB/32): its sum, then an inclusive scan over lanes
    unsigned long long own[NB / 32], ls = 0;
#pragma unroll
    for (int k = 0; k < NB / 32; ++k) {
        const int b = lane * (NB / 32) + k;
        own[k] = (static_cast<unsigned long long>(hw[NB + b]) << 32) + hw[b];
        ls += own[k];
    }
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
    const int J = __ffs(__ballot_sync(0xffffffffu, incl >= target)) - 1;   // lane holding the crossing bin
    unsigned long long run = __shfl_sync(0xffffffffu, incl - ls, J);        // mass of the bins before lane J's
    int cbin = 0;
    unsigned long long above = 0;
#pragma unroll
    for (int k = 0; k < NB / 32; ++k) {   // inside lane J's bins (uniform: broadcast each)
        const unsigned long long bk = __shfl_sync(0xffffffffu, own[k], J);
        if (run < target && run + bk >= target) { cbin = J * (NB / 32) + k; above = run; }
        run += bk;
    }
    // gather the crossing bin's members
    int nm = 0;
    for (int base = 0; base < nc; base += 32) {
        const int i = base + lane;
        const float s = i < nc ? sc[i] : -INFINITY;
        const bool mem = s != -INFINITY && bin_of(s) == cbin;
        const uint32_t bal = __ballot_sync(0xffffffffu, mem);
        const int at = nm + __popc(bal & ((1u << lane) - 1u));
        if (mem && at < kWarpCutMembers) {
            mkey[at] = (static_cast<unsigned long long>(score_key(s)) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
            mmass[at] = score_mass(s, mx);
        }
        nm += __popc(bal);
    }
    if (nm > kWarpCutMembers) return warp_top_p(sc, nc, p, out, node_of);
    __syncwarp();
    const unsigned long long need = target - above;
    // member k is kept iff the mass of the members ordered before it is below `need`;
    // the order is by the key (score, then lower slot first: ~slot)
    int cnt = 0;
    for (int base = 0; base < nc; base += 32) {
        const int i = base + lane;
        const float s = i < nc ? sc[i] : -INFINITY;
        bool keep = false;
        if (s != -INFINITY) {
            const int bn = bin_of(s);
            if (bn < cbin) {
                keep = true;
            } else if (bn == cbin) {
                const unsigned long long myk =
                    (static_cast<unsigned long long>(score_key(s)) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
                unsigned long long before = 0;
                for (int m = 0; m < nm; ++m)
                    if (mkey[m] > myk) before += mmass[m];
                keep = before < need;
            }
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) out[cnt + __popc(bal & ((1u << lane) - 1u))] = node_of(i);
        cnt += __popc(bal);
    }
    return cnt;
}

}  // namespace zha
