// zha_attend.cuh -- exact softmax attention over the routed key set.
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: I(q) = {0} u (union of the kept level-1
// chunks) u C_cur(q), then o(q) = Attn(q, K_I, V_I), "exactly as dense attention
// would" ([EoQ] "Zyphra Hierarchical Attention: The End of Quadratic
// Attention?", A query's path).  The first token is the attention sink ([EoQ],
// How the tree is built and searched).
//
// Decode: the G query heads of one KV head ("group") share the group's key
// blocks, so the group's blocks are gathered once:
//   plan    -- one CTA per group turns the G heads' selected block lists into
//              one ascending list of items (key range + head mask): the union of
//              the blocks, C_cur (merged into its block when that block is in the
//              tree, else a partial range) and the sink (key 0 for the heads whose
//              blocks do not already hold it);
//   attend  -- one CTA per SM; the concatenated item lists of all groups are cut
//              into equal contiguous pieces, one per CTA (split-K, stream-K style).
//              A producer warp streams the piece's K and V rows into shared memory
//              with 1-D bulk async copies (up to 6 stages of 64 rows in flight,
//              full/empty mbarriers); 8 consumer warps keep an online softmax over
//              8 rows of each stage for all G heads.  At the end of each group in
//              its piece the CTA combines its warps into one (max, sum, acc[d])
//              partial per head; the last CTA of a group (atomic counter,
//              self-resetting) merges the group's partials into O.
// Scores are kept in log2 units (q pre-multiplied by scale*log2(e)).
#pragma once

#include "zha_common.cuh"
#include "zha_plan.cuh"

namespace zha {

#ifndef ZHA_ATT_STAGE_BUDGET
#define ZHA_ATT_STAGE_BUDGET (196 * 1024)   // shared memory for the K/V stages of one CTA
#endif
#ifndef ZHA_ATT_CHUNK
#define ZHA_ATT_CHUNK 0
#endif
#ifndef ZHA_ATT_ROTATE
#define ZHA_ATT_ROTATE 1
#endif
constexpr int kAttRows = kItemRowsMax;        // rows per pipeline stage
// stages in flight per CTA: as many 64-row K+V stages as the budget holds, 2..6
template <typename T, int D>
constexpr int att_stages() {
    constexpr int n = ZHA_ATT_STAGE_BUDGET / (2 * 64 * D * static_cast<int>(sizeof(T)));
    return n < 2 ? 2 : (n > 6 ? 6 : n);
}
constexpr int kAttChunk = ZHA_ATT_CHUNK;      // items per round-robin chunk; 0 = one contiguous piece per CTA
constexpr int kSplitMax = 512;        // partials per group (>= the attention grid)

struct AttendArgs {
    const void* K;
    const void* V;
    const void* Q;             // [batch][n_q][Hq][d]
    float* O;                  // [batch][n_q][Hq][d]
    const int2* items;
    const int32_t* n_items;
    float2* part_ml;           // [groups][kSplitMax][G]  (max in log2 units, sum)
    float* part_acc;           // [groups][kSplitMax][G][d]
    uint32_t* counters;        // [groups] partials done, zero between calls
    const float2* pr_ml;       // value summaries: per query row (log2 max, sum) and [d] value sum of
    const float* pr_acc;       //   the nodes routing dropped, one more partial in the merge; else null
    int64_t item_cap, N_cap;
    int groups, Hq, Hkv, n_q;
    float qscale;              // scale * log2(e)
    uint64_t wait_ns;          // bound of a wait on another warp's progress (then ZHA_ERR_TIMEOUT)
};

constexpr int kAttConsumers = 8;                       // consumer warps
constexpr int kAttThreads = 32 * (kAttConsumers + 1);  // + one producer warp
constexpr int kAttRowsPerWarp = kAttRows / kAttConsumers;

struct StageDesc {
    int n_rows;                // -1: no more work
    int group, split;
    int flags;                 // bit 0: last stage of this CTA's piece of the group; bit 1: first stage
    uint32_t heads;            // union of the row masks
    int pad[3];
    uint8_t mask[kAttRows];
};

template <typename T, int D, int G>
struct AttSmem {
    static constexpr int kAttStages = att_stages<T, D>();
    T k[kAttStages][kAttRows][D];
    T v[kAttStages][kAttRows][D];
    T q[kAttStages][G][D];                        // the group's queries, sent with its first stage
    // combine scratch [kAttConsumers/2][G][D]; the group merge reuses it for 2*kSplitMax*G weights
    static constexpr int kRed = (kAttConsumers / 2) * G * D > 2 * kSplitMax * G ? (kAttConsumers / 2) * G * D
                                                                                : 2 * kSplitMax * G;
    float red[kRed];
    float sw[kAttConsumers][2][G][kAttRowsPerWarp];  // scores, per warp and stage of a pair
    float pw[kAttConsumers][2][kAttRowsPerWarp][4];  // probabilities [row][head], per warp and stage
    float cm[kAttConsumers][G], cl[kAttConsumers][G];
    int scan[kAttConsumers + 2];
    StageDesc desc[kAttStages];
    uint64_t full[kAttStages], empty[kAttStages];
    int last_flag, work_split;
    int prefix[1];                                 // [groups + 1] first global item of each group
};

__device__ __forceinline__ void consumer_sync() {   // named barrier of the 8 consumer warps
    asm volatile("bar.sync 1, %0;" ::"n"(kAttConsumers * 32) : "memory");
}

// Split of the concatenated item lists of all groups into chunks of `ch` items;
// chunk j belongs to CTA j mod C.  A CTA's chunks inside one group are
// consecutive in its own order, so it gives at most one partial per group,
// stored at slot = its index; a group has min(C, chunks it spans) partials.
// (Item counts stay below 2^31: 32-bit divisions.)
__device__ __forceinline__ int64_t chunk_items(int64_t I, int C) {
    return kAttChunk > 0 ? kAttChunk : (static_cast<uint32_t>(I) + C - 1) / static_cast<uint32_t>(C);
}
__device__ __forceinline__ int partials_of(int64_t g0, int64_t g1, int64_t ch, int C) {
    const uint32_t uch = static_cast<uint32_t>(ch);
    const int64_t j0 = static_cast<uint32_t>(g0) / uch, j1 = static_cast<uint32_t>(g1 - 1) / uch;
    return static_cast<int>(min(static_cast<int64_t>(C), j1 - j0 + 1));
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kAttThreads, 1) attend_kernel(AttendArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    using Smem = AttSmem<T, D, G>;
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    constexpr int kAttStages = Smem::kAttStages;
    constexpr int VEC = Elem<T>::kVec;       // elements per 16-byte row load (QK layout)
    constexpr int LPR = D / VEC;             // lanes per row
    constexpr int RPW = 32 / LPR;            // rows per load
    constexpr int U = kAttRowsPerWarp / RPW; // loads per lane per stage
    constexpr int NV = U * G;                // partial dots per lane
    constexpr int VD = D / 32;               // PV: dims per lane
    static_assert(G * kAttRowsPerWarp <= 32, "one lane per (head, row) in the softmax");
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    // ---- prefix[g] = first global item of group g (all warps)
    {
        int* pre = sm.prefix;
        int carry = 0;
        for (int base = 0; base < a.groups; base += kAttThreads) {
            const int g = base + tid;
            const int n = g < a.groups ? a.n_items[g] : 0;
            int tot;
            const int x = block_exclusive_scan<kAttConsumers + 1>(n, sm.scan, &tot);
            if (g < a.groups) pre[g] = carry + x;
            carry += tot;
        }
        if (tid == 0) {
            pre[a.groups] = carry;
            for (int i = 0; i < kAttStages; ++i) {
                mbar_init(&sm.full[i], 1);
                mbar_init(&sm.empty[i], kAttConsumers);
            }
            fence_mbar_init();
        }
        __syncthreads();
    }
    const int64_t I = sm.prefix[a.groups];
    const int C = gridDim.x;
    const int64_t ch = I > 0 ? chunk_items(I, C) : 1;

    if (w == kAttConsumers) {
        // ================= producer warp: this CTA's contiguous piece of the item lists, packed
        // into 64-row stages; K/V rows (and each group's queries) sent by 1-D bulk copies.
        int fills = 0;
        bool ok = true;
        auto acquire_slot = [&](int slot) {   // wait until the consumers released this slot
            if (fills >= kAttStages && ok) {
                bool got = true;
                if (lane == 0) got = mbar_wait_bounded(&sm.empty[slot], ((fills / kAttStages) - 1) & 1, a.wait_ns);
                ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!ok && lane == 0) raise_status(ZHA_ERR_TIMEOUT);
            }
        };
        int g = 0;
        int prev_g = -1;
        for (int64_t j = blockIdx.x; j * ch < I && ok; j += C) {
          const int64_t cx_end = min(I, (j + 1) * ch);
          for (int64_t x = j * ch; x < cx_end && ok;) {
            while (sm.prefix[g + 1] <= x) ++g;   // the group holding item x (groups with items only)
            const int64_t g0 = sm.prefix[g], g1 = sm.prefix[g + 1];
            const int64_t seg_end = min(cx_end, g1);
            const int split = blockIdx.x;
            const int i0 = static_cast<int>(x - g0), i1 = static_cast<int>(seg_end - g0);
            // this CTA's run in group g ends with this chunk when its next chunk starts past the group
            const bool run_ends = (j + C) * ch >= g1;
            const bool run_starts = g != prev_g;
            prev_g = g;
            const int s = g / a.Hkv, kv = g % a.Hkv;
            const int64_t kvbase = (static_cast<int64_t>(s) * a.Hkv + kv) * a.N_cap;
            const T* Kb = static_cast<const T*>(a.K) + kvbase * D;
            const T* Vb = static_cast<const T*>(a.V) + kvbase * D;
            const T* Qg = static_cast<const T*>(a.Q) +
                          ((static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G) * D;
            const int2* its = a.items + static_cast<int64_t>(g) * a.item_cap;
            bool first = run_starts;
            // CTAs start at different points of their segments (the order of the keys does not
            // matter to the softmax), so concurrent CTAs do not stream the same address pattern
            const int nseg = i1 - i0;
            const int rot = ZHA_ATT_ROTATE ? static_cast<int>((static_cast<uint32_t>(blockIdx.x) * 2654435761u) % static_cast<uint32_t>(nseg)) : 0;
            for (int part = 0; part < 2; ++part) {
            const int pb0 = part == 0 ? i0 + rot : i0, pb1 = part == 0 ? i1 : i0 + rot;
            for (int base = pb0; base < pb1 && ok; base += 32) {
                const int avail = min(32, pb1 - base);
                int2 it = make_int2(0, 0);
                if (lane < avail) it = its[base + lane];
                int c = it.y & 0xffff;
                if (lane < avail && (c < 1 || c > kAttRows)) { raise_status(ZHA_ERR_INVALID_ARG); c = 0; }
                const uint32_t m = static_cast<uint32_t>(it.y) >> 16;
                int pos = 0;
                while (pos < avail && ok) {
                    int cc = (lane >= pos && lane < avail) ? c : 0;
                    int incl = cc;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    const bool fit = lane >= pos && lane < avail && incl <= kAttRows;
                    const int n_fit = __popc(__ballot_sync(0xffffffffu, fit));
                    const int rows = __shfl_sync(0xffffffffu, incl, pos + n_fit - 1);
                    const int excl = incl - cc;
                    const uint32_t heads = warp_or(fit && cc > 0 ? m : 0u);
                    const bool last = run_ends && pos + n_fit >= avail && base + avail >= pb1 && (part == 1 || rot == 0);
                    const int slot = fills % kAttStages;
                    acquire_slot(slot);
                    if (!ok) break;
                    StageDesc& d = sm.desc[slot];
                    {   // every lane writes the masks of rows 2*lane, 2*lane+1: the item holding row r
                        // is the first fitting lane whose inclusive row count exceeds r, found by a
                        // binary search over the fitting lanes (incl is non-decreasing across them)
                        uint32_t pair = 0;
#pragma unroll
                        for (int k = 0; k < 2; ++k) {
                            const int r = 2 * lane + k;
                            int lo = pos, hi = pos + n_fit - 1;   // incl(hi) = rows > r whenever r < rows
#pragma unroll
                            for (int step = 0; step < 5; ++step) {
                                const int mid = (lo + hi) >> 1;
                                const int im = __shfl_sync(0xffffffffu, incl, mid);
                                if (im > r) hi = mid;
                                else lo = mid + 1 < hi ? mid + 1 : hi;
                            }
                            const uint32_t mo = __shfl_sync(0xffffffffu, m, lo);
                            if (r < rows) pair |= (mo & 0xffu) << (8 * k);
                        }
                        reinterpret_cast<uint16_t*>(d.mask)[lane] = static_cast<uint16_t>(pair);
                    }
                    if (lane == 0) {
                        d.n_rows = rows;
                        d.group = g;
                        d.split = split;
                        d.flags = (last ? 1 : 0) | (first ? 2 : 0);
                        d.heads = heads;
                    }
                    __syncwarp();
                    __threadfence_block();
                    const uint32_t bytes = static_cast<uint32_t>(rows * D * sizeof(T) * 2 + (first ? G * D * sizeof(T) : 0));
                    if (lane == 0) mbar_arrive_expect_tx(&sm.full[slot], bytes);
                    __syncwarp();
                    if (fit && cc > 0) {
                        const int64_t st = it.x;
                        const uint32_t nb = static_cast<uint32_t>(cc * D * sizeof(T));
                        bulk_g2s(&sm.k[slot][excl][0], Kb + st * D, nb, &sm.full[slot]);
                        bulk_g2s(&sm.v[slot][excl][0], Vb + st * D, nb, &sm.full[slot]);
                    }
                    if (first && lane == 0)
                        bulk_g2s(&sm.q[slot][0][0], Qg, static_cast<uint32_t>(G * D * sizeof(T)), &sm.full[slot]);
                    first = false;
                    ++fills;
                    pos += n_fit;
                }
            }
            }
            x = seg_end;
          }
        }
        // the bulk copies of the last stages have landed before this warp leaves (on an abort
        // the consumers may have stopped reading them, and the CTA must not exit with copies
        // in flight); no stage is re-armed before this, so each wait is on its own data phase
        if (lane == 0)
            for (int f = fills > kAttStages ? fills - kAttStages : 0; f < fills; ++f)
                mbar_wait_bounded(&sm.full[f % kAttStages], (f / kAttStages) & 1, kWaitLongNs);
        __syncwarp();
        // sentinel: tells the consumers that no stage follows (not after an abort: a slot still
        // waiting on the consumers must not be re-armed; they give up on their own bound)
        const int slot = fills % kAttStages;
        acquire_slot(slot);
        if (ok && lane == 0) {
            sm.desc[slot].n_rows = -1;
            mbar_arrive(&sm.full[slot]);
        }
        return;
    }

    // ================= consumer warps
    // A warp takes two stages of the same run at a time when it can (the run's last stage
    // may come alone), so every phase below has two independent streams of work.
    float qv[G][VEC];
    float m_run = -INFINITY, l_run = 0.f;      // for head (lane / 8) of this lane
    float acc[G][VD];
    const int sub = lane / LPR, li = lane % LPR;
    const int r0 = w * kAttRowsPerWarp;
    int it = 0;
    bool stop = false;
    while (!stop) {
        const int slotA = it % kAttStages;
        if (!mbar_wait_bounded(&sm.full[slotA], (it / kAttStages) & 1, a.wait_ns)) {
            if (lane == 0) raise_status(ZHA_ERR_TIMEOUT);
            break;
        }
        const StageDesc& dA = sm.desc[slotA];
        const int nA = dA.n_rows;
        if (nA < 0) break;
        const int g = dA.group, split = dA.split;
        int flags = dA.flags;
        uint32_t heads_s[2] = {dA.heads, 0u};
        int slotB = slotA, nB = 0, nst = 1;
        if (!(flags & 1)) {   // not the run's last stage: the next stage belongs to the same run
            slotB = (it + 1) % kAttStages;
            if (!mbar_wait_bounded(&sm.full[slotB], ((it + 1) / kAttStages) & 1, a.wait_ns)) {
                if (lane == 0) raise_status(ZHA_ERR_TIMEOUT);
                break;
            }
            nB = sm.desc[slotB].n_rows;
            if (nB < 0) {        // only after a producer timeout: no second stage
                nB = 0;
                stop = true;
            } else {
                nst = 2;
                flags |= sm.desc[slotB].flags & 1;
                heads_s[1] = sm.desc[slotB].heads;
            }
        }
        if (flags & 2) {   // first stage of this CTA's piece of a group: its queries, fresh state
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x[VEC];
                Elem<T>::load16(&sm.q[slotA][h][li * VEC], x);
#pragma unroll
                for (int e = 0; e < VEC; ++e) qv[h][e] = x[e] * a.qscale;
            }
            m_run = -INFINITY;
            l_run = 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
                for (int e = 0; e < VD; ++e) acc[h][e] = 0.f;
        }
        const int n_s[2] = {nA, nB};
        // this warp's rows of both stages, and the heads each stage needs
        const T* krow_s[2] = {&sm.k[slotA][r0][0], &sm.k[slotB][r0][0]};
        const T* vrow_s[2] = {&sm.v[slotA][r0][0], &sm.v[slotB][r0][0]};
        const uint8_t* mrow_s[2] = {&dA.mask[r0], &sm.desc[slotB].mask[r0]};
        if (r0 < nA || r0 < nB) {
            // QK: lane (sub, li) covers rows r0 + u*RPW + sub, dims [li*VEC, li*VEC+VEC)
            float v[2][NV];
#pragma unroll
            for (int st = 0; st < 2; ++st) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int rl = u * RPW + sub;           // row within the warp's 8
                    float x[VEC];
                    if (r0 + rl < n_s[st]) {
                        Elem<T>::load16(krow_s[st] + rl * D + li * VEC, x);
                    } else {
#pragma unroll
                        for (int e = 0; e < VEC; ++e) x[e] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float dd = 0.f;
                        if ((heads_s[st] >> h) & 1u) {
#pragma unroll
                            for (int e = 0; e < VEC; ++e) dd = fmaf(qv[h][e], x[e], dd);
                        }
                        v[st][h * U + u] = dd;
                    }
                }
            }
            // transpose-reduce over the LPR lanes of a row group (both stages interleaved)
            constexpr int LOG_LPR = LPR == 32 ? 5 : LPR == 16 ? 4 : LPR == 8 ? 3 : 2;
            constexpr int LOG_NV = NV >= 32 ? 5 : NV == 16 ? 4 : NV == 8 ? 3 : NV == 4 ? 2 : NV == 2 ? 1 : 0;
            constexpr int H = LOG_NV < LOG_LPR ? LOG_NV : LOG_LPR;   // halving steps
#pragma unroll
            for (int step = 0; step < LOG_LPR; ++step) {
                const int o = (LPR >> 1) >> step;
                if (step < H) {
                    const int half = NV >> (step + 1);
                    const bool upper = (li & o) != 0;
#pragma unroll
                    for (int i = 0; i < NV / 2; ++i) {
                        if (i < half) {
#pragma unroll
                            for (int st = 0; st < 2; ++st) {
                                const float send = upper ? v[st][i] : v[st][i + half];
                                const float keep = upper ? v[st][i + half] : v[st][i];
                                v[st][i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int st = 0; st < 2; ++st) v[st][0] += __shfl_xor_sync(0xffffffffu, v[st][0], o);
                }
            }
            // the halving steps fix the top H bits of the value index from li's top
            // bits; v[k] then holds index ((li >> low) << (LOG_NV - H)) | k
            {
                constexpr int low = LOG_LPR - H;
                constexpr int NVH = 1 << H;
                if ((li & ((1 << low) - 1)) == 0) {
                    const int vi0 = (li >> low) & (NVH - 1);
#pragma unroll
                    for (int k = 0; k < NV / NVH; ++k) {
                        const int vi = vi0 * (NV / NVH) + k;   // = h * U + u
                        const int h = vi / U, u = vi % U;
#pragma unroll
                        for (int st = 0; st < 2; ++st) sm.sw[w][st][h][u * RPW + sub] = v[st][k];
                    }
                }
            }
            __syncwarp();
            // online softmax over both stages' rows: lane -> (head hh = lane / 8, row rr = lane % 8)
            const int hh = lane / kAttRowsPerWarp, rr = lane % kAttRowsPerWarp;
            const int row = r0 + rr;
            const bool va = hh < G && row < nA && ((mrow_s[0][rr] >> hh) & 1);
            const bool vb = hh < G && row < nB && ((mrow_s[1][rr] >> hh) & 1);
            const float sa = va ? sm.sw[w][0][hh < G ? hh : 0][rr] : -INFINITY;
            const float sb = vb ? sm.sw[w][1][hh < G ? hh : 0][rr] : -INFINITY;
            float mx = fmaxf(sa, sb);
#pragma unroll
            for (int o = 1; o < kAttRowsPerWarp; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float mn = fmaxf(m_run, mx);
            const float alpha = mn == -INFINITY ? 1.f : exp2f(m_run - mn);
            const float pa = va ? exp2f(sa - mn) : 0.f;
            const float pb = vb ? exp2f(sb - mn) : 0.f;
            float ps = pa + pb;
#pragma unroll
            for (int o = 1; o < kAttRowsPerWarp; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l_run = l_run * alpha + ps;
            m_run = mn;
            if (hh < G) {
                sm.pw[w][0][rr][hh] = pa;
                sm.pw[w][1][rr][hh] = pb;
            }
            __syncwarp();
            // PV: lane owns dims [lane*VD, lane*VD+VD) of every head
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float al = __shfl_sync(0xffffffffu, alpha, h * kAttRowsPerWarp);
#pragma unroll
                for (int e = 0; e < VD; ++e) acc[h][e] *= al;
            }
#pragma unroll
            for (int r = 0; r < kAttRowsPerWarp; ++r) {
#pragma unroll
                for (int st = 0; st < 2; ++st) {
                    if (r0 + r < n_s[st]) {
                        float vv[VD];
                        load_n<T, VD>(vrow_s[st] + r * D + lane * VD, vv);
                        const float4 p4 = *reinterpret_cast<const float4*>(&sm.pw[w][st][r][0]);
                        const float pp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                        for (int h = 0; h < G; ++h)
                            if ((heads_s[st] >> h) & 1u)
#pragma unroll
                                for (int e = 0; e < VD; ++e) acc[h][e] = fmaf(pp[h], vv[e], acc[h][e]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) {   // this warp is done with the slot(s)
            mbar_arrive(&sm.empty[slotA]);
            if (nst == 2) mbar_arrive(&sm.empty[slotB]);
        }
        it += nst;

        if (flags & 1) {
            // ---- combine the consumer warps' states into one partial per head
            if (lane % kAttRowsPerWarp == 0 && lane / kAttRowsPerWarp < G) {
                sm.cm[w][lane / kAttRowsPerWarp] = m_run;
                sm.cl[w][lane / kAttRowsPerWarp] = l_run;
            }
            consumer_sync();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float M = -INFINITY;
                for (int ww = 0; ww < kAttConsumers; ++ww) M = fmaxf(M, sm.cm[ww][h]);
                const float f = M == -INFINITY ? 0.f : exp2f(sm.cm[w][h] - M);
#pragma unroll
                for (int e = 0; e < VD; ++e) acc[h][e] *= f;
            }
#pragma unroll
            for (int half = kAttConsumers / 2; half >= 1; half >>= 1) {
                if (w >= half && w < 2 * half)
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) sm.red[((w - half) * G + h) * D + lane * VD + e] = acc[h][e];
                consumer_sync();
                if (w < half)
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) acc[h][e] += sm.red[(w * G + h) * D + lane * VD + e];
                consumer_sync();
            }
            if (w == 0) {
                const int64_t pbase = (static_cast<int64_t>(g) * kSplitMax + split) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float M = -INFINITY, Lsum = 0.f;
                    for (int ww = 0; ww < kAttConsumers; ++ww) M = fmaxf(M, sm.cm[ww][h]);
                    if (M != -INFINITY)
                        for (int ww = 0; ww < kAttConsumers; ++ww) Lsum += sm.cl[ww][h] * exp2f(sm.cm[ww][h] - M);
                    if (lane == 0) a.part_ml[pbase + h] = make_float2(M, Lsum);
#pragma unroll
                    for (int e = 0; e < VD; ++e) a.part_acc[(pbase + h) * D + lane * VD + e] = acc[h][e];
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) {
                    const int sp = partials_of(sm.prefix[g], sm.prefix[g + 1], ch, C);
                    const uint32_t done = atomicAdd(&a.counters[g], 1u);
                    sm.last_flag = done == static_cast<uint32_t>(sp - 1);
                    sm.work_split = sp;
                }
            }
            consumer_sync();
            if (sm.last_flag) {
                // ---- this CTA closes the group: merge its partials into O.  Weights
                // f[k][h] = exp2(m_k - M_h) go to shared memory once; every thread then
                // sums its (head, dim) outputs over the partials with independent loads.
                __threadfence();
                const int sp = sm.work_split;
                const int s = g / a.Hkv, kv = g % a.Hkv;
                const int ct = tid;   // 0 .. 255
                const int64_t pb = static_cast<int64_t>(g) * kSplitMax * G;
                const int slot0 = static_cast<int>((static_cast<uint32_t>(sm.prefix[g]) / static_cast<uint32_t>(ch)) % C);   // partial k sits at slot (slot0+k) % C
                float* fw = sm.red;                      // [kSplitMax][G] weights (red is free here)
                float* fl = fw + kSplitMax * G;          // [kSplitMax][G] partial sums
                for (int x = ct; x < sp * G; x += kAttConsumers * 32) {
                    const int k = x / G, h = x % G;
                    const float2 ml = __ldcg(&a.part_ml[pb + ((slot0 + k) % C) * G + h]);
                    fw[x] = ml.x;
                    fl[x] = ml.y;
                }
                consumer_sync();
                if (w < G) {   // warp h: M_h, the weights, L_h
                    // value summaries: the dropped nodes' partial of this head's query joins the merge
                    const float2 pr = a.pr_ml ? a.pr_ml[(static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + w]
                                              : make_float2(-INFINITY, 0.f);
                    float M = -INFINITY;
                    for (int k = lane; k < sp; k += 32) M = fmaxf(M, fw[k * G + w]);
                    M = fmaxf(warp_max(M), pr.x);
                    float Ls = 0.f;
                    for (int k = lane; k < sp; k += 32) {
                        const float f = M == -INFINITY ? 0.f : exp2f(fw[k * G + w] - M);
                        fw[k * G + w] = f;
                        Ls += f * fl[k * G + w];
                    }
                    Ls = warp_sum(Ls);
                    const float fpr = (M == -INFINITY || pr.x == -INFINITY) ? 0.f : exp2f(pr.x - M);
                    if (lane == 0) {
                        sm.cl[0][w] = fmaf(fpr, pr.y, Ls);
                        sm.cm[0][w] = fpr;
                    }
                }
                consumer_sync();
                for (int x = ct; x < G * D; x += kAttConsumers * 32) {
                    const int h = x / D, e = x % D;
                    const float* src = a.part_acc + (pb + h) * D + e;
                    float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
                    int k = 0;
                    auto at_k = [&](int kk) { return src + static_cast<int64_t>((slot0 + kk) % C) * G * D; };
                    for (; k + 4 <= sp; k += 4) {
                        const float x0 = __ldcg(at_k(k));
                        const float x1 = __ldcg(at_k(k + 1));
                        const float x2 = __ldcg(at_k(k + 2));
                        const float x3 = __ldcg(at_k(k + 3));
                        o0 = fmaf(fw[k * G + h], x0, o0);
                        o1 = fmaf(fw[(k + 1) * G + h], x1, o1);
                        o2 = fmaf(fw[(k + 2) * G + h], x2, o2);
                        o3 = fmaf(fw[(k + 3) * G + h], x3, o3);
                    }
                    for (; k < sp; ++k) o0 = fmaf(fw[k * G + h], __ldcg(at_k(k)), o0);
                    const float Ls = sm.cl[0][h];
                    const int64_t orow = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + h;
                    if (a.pr_acc) o0 = fmaf(sm.cm[0][h], a.pr_acc[orow * D + e], o0);
                    a.O[orow * D + e] = Ls > 0.f ? ((o0 + o1) + (o2 + o3)) / Ls : 0.f;
                }
                if (ct == 0) a.counters[g] = 0u;
                consumer_sync();   // the weights in red are reused by the next combine
            }
        }
    }
}

}  // namespace zha
