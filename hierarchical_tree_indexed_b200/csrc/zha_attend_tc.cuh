// zha_attend_tc.cuh -- decode attention over the routed key set on the
// 5th-generation tensor cores (sm_100a): bf16 K/V/Q, head dim 128, leaf blocks
// of a whole multiple of 64 keys.
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: o(q) = Attn(q, K_I, V_I) over I(q) = {0} u
// (kept level-1 chunks) u C_cur(q), computed exactly as dense attention over
// those keys ([EoQ] "Zyphra Hierarchical Attention: The End of Quadratic
// Attention?", A query's path).
//
// The same work as attend_kernel (zha_attend.cuh) -- the same plan (items of at
// most 64 keys with a head mask, concatenated over the groups and cut into one
// contiguous piece per CTA), the same partials and the same group merge -- with
// the arithmetic of a piece on the tensor cores.  Two items form a pair of 128
// key rows:
//   S^T  = K Q^T     M = 128 keys, N = 16 (the group's G query heads, the rest
//                    ignored), K = 128 dims; A = K tile K-major, B = Q K-major
//   O^T += V^T P^T   M = 128 dims, N = 16, K = 128 keys; A = the V tile read
//                    MN-major (dims contiguous), B = P^T K-major
// P enters as two bf16 parts, hi = bf16(P) in column h and lo = bf16(P - hi)
// in column 4 + h, so P = hi + lo to 2^-18 relative and the output keeps fp32
// accuracy although the tensor cores take bf16; O = column h + column 4 + h.
// Warps 0-3: softmax (thread i owns key row i of a pair, and dimension i of O);
// warp 4: TMA producer; warp 5: TMEM owner and MMA issue (one lane).  The
// online softmax runs in log2 units; O is rescaled lazily, only when a head's
// running max outgrows its reference by 2^8.
// Pieces are cut on a cost axis on which every group starts with kTCGroupCost
// items of virtual cost: a CTA whose piece crosses into another group spends
// that long in the extra epilogue (its softmax warps stall while the group's
// partial is written), so it gets fewer keys and the CTAs end together.
// Every wait is bounded: a timeout raises ZHA_ERR_TIMEOUT, marks the CTA
// aborted, and all later waits return at once, so the kernel always ends.
#pragma once

#include <cuda_bf16.h>

#include "zha_attend.cuh"
#include "zha_umma.cuh"

namespace zha {

constexpr int kTCStages = 3;                                   // pairs of items in flight
constexpr int kTCThreads = 192;
constexpr uint32_t kTCKBytes = 2 * 128 * 128;                  // 128 keys x 128 dims, two 64-dim spans
constexpr uint32_t kTCSpan = 128 * 128;                        // one 64-dim span of a pair
constexpr uint32_t kTCItem = 64 * 128;                         // one item's rows inside a span
constexpr uint32_t kTCQBytes = 2 * 16 * 128;                   // 16 query rows x 128 dims
constexpr uint32_t kTCStageBytes = 2 * kTCKBytes + kTCQBytes;  // K, V, Q of a pair
constexpr uint32_t kTCPBytes = 2 * 16 * 128;                   // P^T: 16 rows x 128 keys
constexpr uint32_t kTCOffP = kTCStages * kTCStageBytes;
constexpr uint32_t kTCOffCtl = kTCOffP + 2 * kTCPBytes;
constexpr uint32_t kTCTmemCols = 64;                           // S: 2 x 16 columns; O: 16 columns at 32
constexpr int kTCGroupCost = 7;                                // a group start on the piece cost axis, in items
constexpr float kTCRescaleLog2 = 8.0f;                         // lazy rescale: P stays below 2^8 between rescales

struct TcDesc {
    int n0, n1;                // keys of the pair's items (n1 = 0: one item); n0 < 0: no more work
    uint32_t heads0, heads1;   // head masks of the two items
    int group, split;
    int flags;                 // bit 0: last pair of this CTA's piece of the group; bit 1: first pair;
                               // bit 2: last pair of the CTA's whole piece
    int pad;
};

struct TcCtl {
    uint64_t kv_full[kTCStages];   // TMA -> all: K, V, Q of the pair landed (and its descriptor written)
    uint64_t kv_empty[kTCStages];  // MMA -> TMA: P V of the pair completed
    uint64_t s_full[2];            // MMA -> softmax: S^T of pair g in TMEM buffer g & 1
    uint64_t s_free[2];            // softmax -> MMA: S^T buffer read
    uint64_t p_full[2];            // softmax -> MMA: P^T of pair g written, O rescaled
    uint64_t o_done[2];            // MMA -> softmax: P V of pair g (and every MMA before it) completed
    uint64_t mx[2];                // softmax warps: pair maxima exchanged
    uint64_t ep[3];                // softmax warps: partial sums exchanged / partial stored / merge decided
    uint64_t mg[2];                // softmax warps: a merge's (max, sum) gathered (merge in mid-piece) / weights formed
    uint64_t mgb;                  // bulk copies: a merge's partials landed in the stage buffers
    uint64_t pre_ready;            // producer -> softmax: prefix[] written
    uint64_t fin;                  // MMA lane: every MMA it issued completed
    TcDesc desc[kTCStages];
    uint32_t tmem;
    int abort;
    int last_flag, sp, sp0;
    uint64_t wait_ns;              // bound of a wait on another warp's progress
    int red[2][4][4];              // [pair parity][warp][head] order-mapped maxima
    float lsum[4][4];              // [warp][head] softmax sums
    float mL[4];                   // [head] a merge's total sum, the dropped nodes' partial included
    float mPr[4];                  // [head] a merge's weight of the dropped nodes' partial (value summaries)
    int prefix[1];                 // [groups + 1] first global item of each group; then the merge's
                                   // (max, sum) -> (weight, sum) of every partial, float2 [grid][4]
};

__host__ __device__ constexpr size_t tc_merge_offset(int groups) {   // from the start of TcCtl, 8-aligned
    return (sizeof(TcCtl) + sizeof(int) * static_cast<size_t>(groups) + 7) & ~static_cast<size_t>(7);
}
__host__ __device__ constexpr size_t tc_smem_bytes(int groups, int grid) {
    return kTCOffCtl + tc_merge_offset(groups) + sizeof(float2) * 4 * static_cast<size_t>(grid) + 1024;   // + alignment slack
}

// Bounded wait; a timeout is recorded once and later waits of the CTA return at once.
__device__ __forceinline__ bool twait(uint64_t* bar, uint32_t parity, TcCtl* ctl) {
    if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
    if (mbar_wait_bounded(bar, parity, ctl->wait_ns)) return true;
    *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
    raise_status(ZHA_ERR_TIMEOUT);
    return false;
}
__device__ __forceinline__ bool tc_aborted(TcCtl* ctl) { return *reinterpret_cast<volatile int*>(&ctl->abort) != 0; }

// The piece cost axis: group g's items occupy [cost_start(g), cost_start(g) + n_g), each
// group preceded by kTCGroupCost items of virtual cost; CTA j covers [j cc, (j + 1) cc).
// Costs stay below 2^31 (32-bit arithmetic), like the item counts.
__device__ __forceinline__ uint32_t tc_cost_chunk(int64_t I, int groups, int C) {
    const uint32_t Ic = static_cast<uint32_t>(I) + static_cast<uint32_t>(kTCGroupCost * groups);
    return I > 0 ? (Ic + static_cast<uint32_t>(C) - 1) / static_cast<uint32_t>(C) : 1u;
}
__device__ __forceinline__ uint32_t tc_cost_start(const int* prefix, int g) {
    return static_cast<uint32_t>(prefix[g]) + static_cast<uint32_t>(kTCGroupCost * (g + 1));
}

// Order-preserving map of floats (no NaN) to int, for the integer warp max.
__device__ __forceinline__ int ord_of(float x) {
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float of_ord(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

template <int G>
__global__ void __launch_bounds__(kTCThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, AttendArgs a) {
    constexpr int D = 128;
    static_assert(G >= 1 && G <= 4, "at most 4 query heads per KV head");
    extern __shared__ __align__(1024) unsigned char tc_smem[];
    const uint32_t raw_s = smem_addr(tc_smem);
    unsigned char* base = tc_smem + (((raw_s + 1023u) & ~1023u) - raw_s);
    unsigned char* sP = base + kTCOffP;
    TcCtl* ctl = reinterpret_cast<TcCtl*>(base + kTCOffCtl);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    auto stage = [&](int s) { return base + static_cast<uint32_t>(s) * kTCStageBytes; };

    // ---- barriers; TMEM; P^T rows 8..15 stay zero.  The group prefix is the producer's
    // first job (published through pre_ready), so its first loads go out without a block scan.
    if (tid == 0) {
        for (int i = 0; i < kTCStages; ++i) {
            mbar_init(&ctl->kv_full[i], 1);
            mbar_init(&ctl->kv_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->s_full[i], 1);
            mbar_init(&ctl->s_free[i], 128);
            mbar_init(&ctl->p_full[i], 128);
            mbar_init(&ctl->o_done[i], 1);
            mbar_init(&ctl->mx[i], 4);
        }
        mbar_init(&ctl->ep[0], 4);
        mbar_init(&ctl->ep[1], 4);
        mbar_init(&ctl->ep[2], 1);
        mbar_init(&ctl->mg[0], 4);
        mbar_init(&ctl->mg[1], 4);
        mbar_init(&ctl->mgb, 1);
        mbar_init(&ctl->pre_ready, 1);
        mbar_init(&ctl->fin, 1);
        fence_mbar_init();
        ctl->abort = 0;
        ctl->wait_ns = a.wait_ns;
        umma::prefetch_tensormap(&tmK);
        umma::prefetch_tensormap(&tmV);
        umma::prefetch_tensormap(&tmQ);
    }
    for (int x = tid; x < static_cast<int>(2 * kTCPBytes / 16); x += kTCThreads)
        reinterpret_cast<uint4*>(sP)[x] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 5) {
        umma::tmem_alloc(&ctl->tmem, kTCTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem;
    const int C = gridDim.x;

    if (warp == 4) {
        // ================= TMA producer: this CTA's piece, two items per pair
        // prefix[g] = first global item of group g: lane l sums a run of groups, a warp scan
        // places the runs, lane l writes its run's prefixes
        const int per = (a.groups + 31) / 32;
        const int r0 = min(a.groups, lane * per), r1 = min(a.groups, r0 + per);
        int run = 0;
#pragma unroll 4
        for (int g = r0; g < r1; ++g) run += a.n_items[g];
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int acc = incl - run;
        for (int g = r0; g < r1; ++g) {
            ctl->prefix[g] = acc;
            acc += a.n_items[g];
        }
        const int64_t I = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0) ctl->prefix[a.groups] = static_cast<int>(I);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->pre_ready);
        const uint32_t cc = tc_cost_chunk(I, a.groups, C);   // cost per CTA: one contiguous piece each
        int fills = 0;     // pairs posted (lane 0's count is the one used)
        bool ok = true;
        auto acquire = [&](int f) -> bool {
            return f < kTCStages || twait(&ctl->kv_empty[f % kTCStages], ((f / kTCStages) - 1) & 1, ctl);
        };
        if (I > 0) {
            const uint32_t c0 = static_cast<uint32_t>(blockIdx.x) * cc, c1 = c0 + cc;
            int g = 0;
            while (g < a.groups && tc_cost_start(ctl->prefix, g) + (ctl->prefix[g + 1] - ctl->prefix[g]) <= c0) ++g;
            int g_fin = -1;   // the piece's last group with keys in it
            for (int x = g; x < a.groups && tc_cost_start(ctl->prefix, x) < c1; ++x) {
                const uint32_t cs = tc_cost_start(ctl->prefix, x);
                if ((c0 > cs ? static_cast<int>(c0 - cs) : 0) < min(ctl->prefix[x + 1] - ctl->prefix[x], static_cast<int>(c1 - cs)))
                    g_fin = x;
            }
            for (; g < a.groups && tc_cost_start(ctl->prefix, g) < c1 && ok; ++g) {
                const uint32_t cs = tc_cost_start(ctl->prefix, g);
                const int ng = ctl->prefix[g + 1] - ctl->prefix[g];
                const int i0 = c0 > cs ? static_cast<int>(c0 - cs) : 0;
                const int i1 = min(ng, static_cast<int>(c1 - cs));
                if (i0 >= i1) continue;
                const int nseg = i1 - i0;
                // CTAs start at different points of their segments (the order of the keys does
                // not matter to the softmax), so concurrent CTAs stream different address patterns
                const int rot = static_cast<int>((static_cast<uint32_t>(blockIdx.x) * 2654435761u) %
                                                 static_cast<uint32_t>(nseg));
                const int s = g / a.Hkv, kv = g % a.Hkv;
                const int qrow = (s * a.n_q + (a.n_q - 1)) * a.Hq + kv * G;
                const int2* its = a.items + static_cast<int64_t>(g) * a.item_cap;
                auto item_at = [&](int v) {   // the segment's v-th item in this CTA's order
                    v += rot;
                    if (v >= nseg) v -= nseg;
                    return its[i0 + v];
                };
                int2 nx = make_int2(0, 0);    // the next batch of 32 items
                if (lane < nseg) nx = item_at(lane);
                for (int vb = 0; vb < nseg && ok; vb += 32) {
                    const int avail = min(32, nseg - vb);
                    const int2 it = nx;
                    nx = make_int2(0, 0);
                    if (vb + 32 + lane < nseg) nx = item_at(vb + 32 + lane);
                    int c = it.y & 0xffff;
                    if (lane < avail && (c < 1 || c > 64)) {
                        raise_status(ZHA_ERR_INVALID_ARG);
                        c = 0;
                    }
                    const uint32_t m = static_cast<uint32_t>(it.y) >> 16;
                    for (int p = 0; p < avail; p += 2) {
                        const bool two = p + 1 < avail;
                        const int q1 = two ? p + 1 : p;
                        const int st0 = __shfl_sync(0xffffffffu, it.x, p);
                        const int st1 = __shfl_sync(0xffffffffu, it.x, q1);
                        const int c0 = __shfl_sync(0xffffffffu, c, p);
                        const int c1 = two ? __shfl_sync(0xffffffffu, c, q1) : 0;
                        const uint32_t m0 = __shfl_sync(0xffffffffu, m, p);
                        const uint32_t m1 = __shfl_sync(0xffffffffu, m, q1);
                        int posted = 0;
                        if (lane == 0 && acquire(fills)) {
                            const int slot = fills % kTCStages;
                            TcDesc& d = ctl->desc[slot];
                            d.n0 = c0;
                            d.n1 = c1;
                            d.heads0 = c0 > 0 ? m0 : 0u;
                            d.heads1 = c1 > 0 ? m1 : 0u;
                            d.group = g;
                            d.split = blockIdx.x;
                            d.flags = (vb + p + 2 >= nseg ? (g == g_fin ? 5 : 1) : 0) | (vb + p == 0 ? 2 : 0);
                            unsigned char* sb = stage(slot);
                            uint64_t* bar = &ctl->kv_full[slot];
                            const uint32_t bytes = (c0 > 0 ? 2 * kTCSpan : 0u) + (c1 > 0 ? 2 * kTCSpan : 0u) + kTCQBytes;
                            mbar_arrive_expect_tx(bar, bytes);
                            // an item's 64 rows from its first key (rows past the cache's end
                            // read as zeros), both 64-dim spans, K and V
                            if (c0 > 0) {
                                umma::tma_load_3d(sb, &tmK, 0, st0, g, bar);
                                umma::tma_load_3d(sb + kTCSpan, &tmK, 64, st0, g, bar);
                                umma::tma_load_3d(sb + kTCKBytes, &tmV, 0, st0, g, bar);
                                umma::tma_load_3d(sb + kTCKBytes + kTCSpan, &tmV, 64, st0, g, bar);
                            }
                            if (c1 > 0) {
                                umma::tma_load_3d(sb + kTCItem, &tmK, 0, st1, g, bar);
                                umma::tma_load_3d(sb + kTCSpan + kTCItem, &tmK, 64, st1, g, bar);
                                umma::tma_load_3d(sb + kTCKBytes + kTCItem, &tmV, 0, st1, g, bar);
                                umma::tma_load_3d(sb + kTCKBytes + kTCSpan + kTCItem, &tmV, 64, st1, g, bar);
                            }
                            umma::tma_load_2d(sb + 2 * kTCKBytes, &tmQ, 0, qrow, bar);
                            umma::tma_load_2d(sb + 2 * kTCKBytes + kTCQBytes / 2, &tmQ, 64, qrow, bar);
                            posted = 1;
                        }
                        ok = __shfl_sync(0xffffffffu, posted, 0) != 0;
                        if (!ok) break;
                        ++fills;
                    }
                }
            }
        }
        if (lane == 0) {
            if (ok && acquire(fills)) {   // sentinel: no pair follows
                ctl->desc[fills % kTCStages].n0 = -1;
                mbar_arrive(&ctl->kv_full[fills % kTCStages]);
                ++fills;
            }
            // the loads of the last pairs have landed before the CTA may exit (the slot the
            // sentinel re-armed held a pair the MMAs had consumed, so its data was in)
            for (int f = fills > kTCStages ? fills - kTCStages : 0; f < fills; ++f)
                mbar_wait_bounded(&ctl->kv_full[f % kTCStages], (f / kTCStages) & 1, kWaitLongNs);
        }
    } else if (warp == 5) {
        // ================= MMA issue (one lane): S^T and P V of the pairs in order
        if (lane == 0) {
            constexpr uint32_t kIdS = umma::idesc_bf16_ab(128, 16, false, false);
            constexpr uint32_t kIdO = umma::idesc_bf16_ab(128, 16, true, false);
            const uint32_t tO = tmem + 32;
            auto pv = [&](uint32_t h) {   // P^T of pair h is written
                const int slot = static_cast<int>(h % kTCStages);
                umma::fence_after_sync();
                const bool first = (ctl->desc[slot].flags & 2) != 0;
                const unsigned char* vb = stage(slot) + kTCKBytes;
                const unsigned char* pb = sP + (h & 1u) * kTCPBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {   // 16 keys per step
                    const uint64_t ad = umma::desc_sw128(smem_addr(vb + kk * 2048), kTCSpan, 1024);
                    const uint64_t bd = umma::desc_sw128(smem_addr(pb + (kk >> 2) * 2048 + (kk & 3) * 32), 16, 1024);
                    umma::mma_bf16(tO, ad, bd, kIdO, (kk > 0 || !first) ? 1u : 0u);
                }
                umma::commit(&ctl->o_done[h & 1u]);
                umma::commit(&ctl->kv_empty[slot]);
            };
            // S^T of pair gs as soon as its tiles landed and its TMEM buffer is free; P V of pair
            // gp as soon as its softmax is done -- polled, so that neither waits on the other and
            // a pair's stage is released right after its own softmax.
            uint32_t gs = 0, gp = 0;
            bool no_more = false;
            uint64_t t_last = global_timer_ns();
            for (uint32_t idle = 0;;) {
                bool progress = false;
                if (!no_more) {
                    const int slot = static_cast<int>(gs % kTCStages);
                    if (mbar_test_wait(&ctl->kv_full[slot], (gs / kTCStages) & 1u)) {
                        if (ctl->desc[slot].n0 < 0) {
                            no_more = true;
                        } else if (gs < 2 || mbar_test_wait(&ctl->s_free[gs & 1u], ((gs - 2) >> 1) & 1u)) {
                            umma::fence_after_sync();
                            const unsigned char* kb = stage(slot);
                            const unsigned char* qb = kb + 2 * kTCKBytes;
                            const uint32_t tS = tmem + (gs & 1u) * 16;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {   // 16 dims per step
                                const uint64_t ad = umma::desc_sw128(smem_addr(kb + (kk >> 2) * kTCSpan + (kk & 3) * 32), 16, 1024);
                                const uint64_t bd = umma::desc_sw128(smem_addr(qb + (kk >> 2) * (kTCQBytes / 2) + (kk & 3) * 32), 16, 1024);
                                umma::mma_bf16(tS, ad, bd, kIdS, kk > 0 ? 1u : 0u);
                            }
                            umma::commit(&ctl->s_full[gs & 1u]);
                            ++gs;
                            progress = true;
                        }
                    }
                }
                if (gp < gs && mbar_test_wait(&ctl->p_full[gp & 1u], (gp >> 1) & 1u)) {
                    pv(gp);
                    ++gp;
                    progress = true;
                }
                if (no_more && gp == gs) break;
                if (progress) {
                    idle = 0;
                    t_last = global_timer_ns();
                } else if ((++idle & 1023u) == 0) {
                    if (tc_aborted(ctl)) break;
                    if (global_timer_ns() - t_last > ctl->wait_ns) {
                        *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
                        raise_status(ZHA_ERR_TIMEOUT);
                        break;
                    }
                }
            }
            umma::commit(&ctl->fin);
            mbar_wait_bounded(&ctl->fin, 0, kWaitLongNs);   // every MMA issued has completed
        }
    } else {
        // ================= softmax warps 0-3
        const int i = tid;   // key row i of each pair; dimension i of O
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        float m_ref[4], l[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            m_ref[h] = -INFINITY;
            l[h] = 0.f;
        }
        twait(&ctl->pre_ready, 0, ctl);   // the group prefix (first read by an epilogue)
        const uint32_t cc = tc_cost_chunk(ctl->prefix[a.groups], a.groups, C);
        uint32_t e = 0, nm = 0, nmg = 0;   // epilogues, merges, merges from global memory
        float2* mbuf = reinterpret_cast<float2*>(reinterpret_cast<unsigned char*>(ctl) + tc_merge_offset(a.groups));
        for (uint32_t g = 0;; ++g) {
            if (tc_aborted(ctl)) break;
            const int slot = static_cast<int>(g % kTCStages);
            twait(&ctl->kv_full[slot], (g / kTCStages) & 1u, ctl);
            if (tc_aborted(ctl)) break;
            const TcDesc d = ctl->desc[slot];
            if (d.n0 < 0) break;
            const bool first = (d.flags & 2) != 0, last = (d.flags & 1) != 0;
            const int n = i < 64 ? d.n0 : d.n1;
            const uint32_t hm = i < 64 ? d.heads0 : d.heads1;
            const bool vrow = (i & 63) < n;
            if (first) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    m_ref[h] = -INFINITY;
                    l[h] = 0.f;
                }
            }
            if (!vrow) {   // the tensor cores read every V row of the pair: rows outside the items are zeroed
                unsigned char* vr = stage(slot) + kTCKBytes + i * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    reinterpret_cast<uint4*>(vr)[c] = make_uint4(0u, 0u, 0u, 0u);
                    reinterpret_cast<uint4*>(vr + kTCSpan)[c] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            twait(&ctl->s_full[g & 1u], (g >> 1) & 1u, ctl);
            umma::fence_after_sync();
            float sv[4];
            umma::tmem_ld4(tmem + (g & 1u) * 16 + lane_base, sv);
            umma::fence_before_sync();
            mbar_arrive(&ctl->s_free[g & 1u]);
#pragma unroll
            for (int h = 0; h < 4; ++h) sv[h] = (h < G && vrow && ((hm >> h) & 1u)) ? sv[h] * a.qscale : -INFINITY;
            // the pair's max per head over the four warps
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int k = __reduce_max_sync(0xffffffffu, ord_of(sv[h]));
                if (lane == 0) ctl->red[g & 1u][warp][h] = k;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->mx[g & 1u]);
            twait(&ctl->mx[g & 1u], (g >> 1) & 1u, ctl);
            bool resc = false;
            float alpha[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                int k = ctl->red[g & 1u][0][h];
#pragma unroll
                for (int ww = 1; ww < 4; ++ww) k = max(k, ctl->red[g & 1u][ww][h]);
                const float tmax = of_ord(k);
                alpha[h] = 1.f;
                if (tmax > m_ref[h] + kTCRescaleLog2) {   // lazy: move the reference only by more than 2^8
                    if (m_ref[h] != -INFINITY) {
                        alpha[h] = exp2f(m_ref[h] - tmax);
                        l[h] *= alpha[h];
                        resc = true;
                    }
                    m_ref[h] = tmax;
                }
            }
            // P V of pair g - 2 has read the P buffer this pair writes
            if (g >= 2) twait(&ctl->o_done[g & 1u], ((g - 2) >> 1) & 1u, ctl);
            if (resc) {   // uniform: every thread sees the same maxima; never on a piece's first pair
                twait(&ctl->o_done[(g - 1) & 1u], ((g - 1) >> 1) & 1u, ctl);
                umma::fence_after_sync();
                float o[8];
                umma::tmem_ld8(tmem + 32 + lane_base, o);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    o[h] *= alpha[h];
                    o[4 + h] *= alpha[h];
                }
                umma::tmem_st8(tmem + 32 + lane_base, o);
            }
            // P^T, K-major 128-byte swizzle: row n (head part), key i -> span i / 64, chunk (i % 64) / 8
            unsigned char* pb = sP + (g & 1u) * kTCPBytes + (i >> 6) * 2048;
            const int kc = (i & 63) >> 3, kb = (i & 7) * 2;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float p = sv[h] == -INFINITY ? 0.f : exp2f(sv[h] - m_ref[h]);
                l[h] += p;
                const __nv_bfloat16 hi = __float2bfloat16_rn(p);
                const __nv_bfloat16 lo = __float2bfloat16_rn(p - __bfloat162float(hi));
                *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((kc ^ h) << 4) + kb) = hi;
                *reinterpret_cast<__nv_bfloat16*>(pb + (4 + h) * 128 + ((kc ^ (4 + h)) << 4) + kb) = lo;
            }
            umma::fence_proxy_async_smem();   // P^T and the zeroed V rows, for the tensor cores
            umma::fence_before_sync();
            mbar_arrive(&ctl->p_full[g & 1u]);

            if (last) {
                // ---- this CTA's partial of the group: (max, sum) per head and O^T, unnormalised
                twait(&ctl->o_done[g & 1u], (g >> 1) & 1u, ctl);
                umma::fence_after_sync();
                float o[8];
                umma::tmem_ld8(tmem + 32 + lane_base, o);
                umma::fence_before_sync();
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float sum = warp_sum(l[h]);
                    if (lane == 0) ctl->lsum[warp][h] = sum;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->ep[0]);
                twait(&ctl->ep[0], e & 1u, ctl);
                const int grp = d.group, split = d.split;
                const int64_t pbase = (static_cast<int64_t>(grp) * kSplitMax + split) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float L = (ctl->lsum[0][h] + ctl->lsum[1][h]) + (ctl->lsum[2][h] + ctl->lsum[3][h]);
                    if (i == 0) a.part_ml[pbase + h] = make_float2(m_ref[h], L);
                    a.part_acc[(pbase + h) * D + i] = o[h] + o[4 + h];
                }
                // the CTA's stores are ordered before thread 0's count by the barrier; the count's
                // release publishes them at GPU scope, and its acquire makes the other CTAs'
                // partials visible to this CTA (through the barrier that follows) when it merges
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->ep[1]);
                if (i == 0) {
                    twait(&ctl->ep[1], e & 1u, ctl);
                    // the CTAs whose pieces meet the group's items: slots j0 .. j1
                    const uint32_t cs = tc_cost_start(ctl->prefix, grp);
                    const int j0 = static_cast<int>(cs / cc);
                    const int j1 = static_cast<int>((cs + (ctl->prefix[grp + 1] - ctl->prefix[grp]) - 1) / cc);
                    const int sp = j1 - j0 + 1;
                    const uint32_t done = atomic_add_acq_rel_gpu(&a.counters[grp], 1u);
                    ctl->last_flag = done == static_cast<uint32_t>(sp - 1);
                    ctl->sp = sp;
                    ctl->sp0 = j0;
                    mbar_arrive(&ctl->ep[2]);
                }
                twait(&ctl->ep[2], e & 1u, ctl);
                if (ctl->last_flag) {
                    // ---- this CTA closes the group: merge its partials (slots sp0 .. sp0 + sp - 1,
                    // one contiguous run of the workspace) into O.  After the CTA's last pair the
                    // stage buffers are idle, and two bulk copies bring the run's (max, sum) pairs
                    // and accumulators into them; a merge in mid-piece (rare) gathers the pairs
                    // into shared memory and reads the accumulators from global memory.  Warp h
                    // forms head h's weights 2^(m_k - M_h) in place and the total sum; then thread
                    // i sums dimension i over the partials with shared-memory loads and FMAs only.
                    // The loops stay rolled: this code runs once per group, from a cold
                    // instruction cache.
                    const int sp = ctl->sp;
                    const int s = grp / a.Hkv, kv = grp % a.Hkv;
                    const int64_t pb0 = (static_cast<int64_t>(grp) * kSplitMax + ctl->sp0) * G;   // partial k, head h: entry pb0 + k G + h
                    const int64_t orow0 = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G;
                    const uint32_t acc_bytes = static_cast<uint32_t>(sp * G * D) * 4u, ml_bytes = static_cast<uint32_t>(sp * G) * 8u;
                    const bool staged = (d.flags & 4) != 0 && acc_bytes + ml_bytes <= kTCStages * kTCStageBytes;
                    const float* sacc = reinterpret_cast<const float*>(stage(0));
                    float2* sml = staged ? reinterpret_cast<float2*>(stage(0) + acc_bytes) : mbuf;
                    // value summaries: the dropped nodes' partial of each head's query joins the merge
                    float pa[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) pa[h] = a.pr_acc ? a.pr_acc[(orow0 + h) * D + i] : 0.f;
                    if (staged) {
                        if (i == 0) {
                            // the count's acquire made the partials visible to this thread; the
                            // bulk copies read them through the async proxy
                            umma::fence_proxy_async_global();
                            mbar_arrive_expect_tx(&ctl->mgb, acc_bytes + ml_bytes);
                            bulk_g2s(stage(0), a.part_acc + pb0 * D, acc_bytes, &ctl->mgb);
                            bulk_g2s(stage(0) + acc_bytes, a.part_ml + pb0, ml_bytes, &ctl->mgb);
                        }
                        twait(&ctl->mgb, (nm - nmg) & 1u, ctl);
                    } else {
                        for (int x = i; x < sp * G; x += 128) mbuf[x] = __ldcg(&a.part_ml[pb0 + x]);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->mg[0]);
                        twait(&ctl->mg[0], nmg & 1u, ctl);
                        ++nmg;
                    }
                    if (warp < G) {
                        const int h = warp;
                        const float2 pr = a.pr_ml ? a.pr_ml[orow0 + h] : make_float2(-INFINITY, 0.f);
                        float M = pr.x;
                        for (int k = lane; k < sp; k += 32) M = fmaxf(M, sml[k * G + h].x);
                        M = warp_max(M);
                        float Ls = 0.f;
                        for (int k = lane; k < sp; k += 32) {
                            const float2 ml = sml[k * G + h];
                            const float f = M == -INFINITY ? 0.f : exp2f(ml.x - M);
                            sml[k * G + h].x = f;
                            Ls = fmaf(f, ml.y, Ls);
                        }
                        Ls = warp_sum(Ls);
                        const float fpr = (M == -INFINITY || pr.x == -INFINITY) ? 0.f : exp2f(pr.x - M);
                        if (lane == 0) {
                            ctl->mL[h] = fmaf(fpr, pr.y, Ls);
                            ctl->mPr[h] = fpr;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl->mg[1]);
                    twait(&ctl->mg[1], nm & 1u, ctl);
                    float o[G];
#pragma unroll
                    for (int h = 0; h < G; ++h) o[h] = ctl->mPr[h] * pa[h];
                    if (staged) {
#pragma unroll 4
                        for (int k = 0; k < sp; ++k)
#pragma unroll
                            for (int h = 0; h < G; ++h) o[h] = fmaf(sml[k * G + h].x, sacc[(k * G + h) * D + i], o[h]);
                    } else {
#pragma unroll 4
                        for (int k = 0; k < sp; ++k)
#pragma unroll
                            for (int h = 0; h < G; ++h)
                                o[h] = fmaf(sml[k * G + h].x, __ldcg(a.part_acc + (pb0 + k * G + h) * D + i), o[h]);
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float Ls = ctl->mL[h];
                        a.O[(orow0 + h) * D + i] = Ls > 0.f ? o[h] / Ls : 0.f;
                    }
                    ++nm;
                    if (i == 0) a.counters[grp] = 0u;
                }
                ++e;
            }
        }
    }
    __syncthreads();
    if (warp == 5) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kTCTmemCols);
    }
}

}  // namespace zha
