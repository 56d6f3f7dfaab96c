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
//   attend  -- persistent split-K kernel: each CTA streams its items' K and V rows
//              into shared memory with 1-D bulk async copies (3-stage mbarrier
//              pipeline, 64 rows per stage), and every warp keeps an online
//              softmax over its 8 rows of each stage for all G heads;
//              at the end of a split the warps combine, the CTA writes one
//              (max, sum, acc[d]) partial per head, and the last CTA of a group
//              (atomic counter, self-resetting) merges the group's partials into O.
// Scores are kept in log2 units (q pre-multiplied by scale*log2(e)).
#pragma once

#include "zha_common.cuh"

namespace zha {

constexpr int kAttThreads = 256;
constexpr int kAttWarps = 8;
constexpr int kAttRows = 64;          // rows per pipeline stage
constexpr int kAttStages = 3;
constexpr int kAttRowsPerWarp = kAttRows / kAttWarps;
constexpr int kSplitMax = 256;        // partials per group
constexpr int kItemsPerSplitMin = 4;
constexpr int kPlanThreads = 512;

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

// One CTA per (sequence, KV head).
__global__ void __launch_bounds__(kPlanThreads) plan_decode_kernel(PlanArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem_raw);   // [G][words]
    __shared__ int scan[kPlanThreads / 32 + 1];
    const int g = blockIdx.x, s = g / a.Hkv, kv = g % a.Hkv, tid = threadIdx.x;
    const int G = a.G;
    const uint32_t all = (1u << G) - 1u;
    const int64_t N = a.N[s], Ntree = a.n_tree[s];
    if (N < 1 || N > a.N_cap || Ntree > N) {
        if (tid == 0) { raise_status(ZHA_ERR_INVALID_ARG); a.n_items[g] = 0; a.rows[g] = 0; }
        return;
    }
    const int64_t t = N - 1;
    const int64_t n1 = Ntree / a.B;
    const int64_t words = (n1 + 31) / 32;
    for (int64_t i = tid; i < G * words; i += kPlanThreads) bits[(i / words) * a.words + i % words] = 0u;
    __syncthreads();
    for (int h = 0; h < G; ++h) {
        const int64_t row = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + h;
        const int cnt = min(a.sel_count[row], a.sel_cap);
        const int32_t* sl = a.sel + row * a.sel_cap;
        for (int i = tid; i < cnt; i += kPlanThreads) {
            const int32_t blk = sl[i];
            if (blk >= 0 && blk < n1) atomicOr(&bits[h * a.words + (blk >> 5)], 1u << (blk & 31));
        }
    }
    const int64_t cb = min(t / a.B, n1);   // C_cur = [cb*B, t]
    if (tid < G && cb < n1) atomicOr(&bits[tid * a.words + (cb >> 5)], 1u << (cb & 31));
    __syncthreads();
    // compaction of the union, ascending: thread owns words [w0, w1)
    const int64_t per = (words + kPlanThreads - 1) / kPlanThreads;
    const int64_t w0 = min(words, tid * per), w1 = min(words, w0 + per);
    int c = 0;
    for (int64_t wd = w0; wd < w1; ++wd) {
        uint32_t o = 0;
        for (int h = 0; h < G; ++h) o |= bits[h * a.words + wd];
        c += __popc(o);
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
            out[pos++] = make_item((wd * 32 + bit) * a.B, a.B, m);
        }
    }
    if (tid == 0) {
        int n = total;
        int64_t rows = static_cast<int64_t>(total) * a.B;
        if (n1 >= 1) {   // sink: key 0 for the heads whose block 0 is not in the union
            uint32_t m0 = 0;
            for (int h = 0; h < G; ++h) m0 |= (bits[h * a.words] & 1u) << h;
            if ((m0 & all) != all) { out[n++] = make_item(0, 1, all & ~m0); rows += 1; }
        }
        if (cb == n1)   // C_cur past the last leaf block: the keys [n1*B, t], 64 at a time
            for (int64_t st = cb * a.B; st <= t && n < a.item_cap; st += kAttRows) {
                const int c = static_cast<int>(t - st + 1 < kAttRows ? t - st + 1 : kAttRows);
                out[n++] = make_item(st, c, all);
                rows += c;
            }
        a.n_items[g] = n;
        a.rows[g] = static_cast<int32_t>(rows);
    }
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
    const int64_t cnt = (n + kAttRows - 1) / kAttRows;
    const uint32_t all = (1u << G) - 1u;
    for (int64_t i = threadIdx.x; i < cnt; i += blockDim.x)
        items[g * item_cap + i] = make_item(i * kAttRows, static_cast<int>(n - i * kAttRows < kAttRows ? n - i * kAttRows : kAttRows), all);
    if (threadIdx.x == 0) n_items[g] = static_cast<int32_t>(cnt);
}

struct AttendArgs {
    const void* K;
    const void* V;
    const void* Q;             // [batch][n_q][Hq][d]
    float* O;                  // [batch][n_q][Hq][d]
    const int2* items;
    const int32_t* n_items;
    float2* part_ml;           // [groups][kSplitMax][G]  (max in log2 units, sum)
    float* part_acc;           // [groups][kSplitMax][G][d]
    uint32_t* counters;        // [groups], zero between calls
    int64_t item_cap, N_cap;
    int groups, Hq, Hkv, n_q;
    float qscale;              // scale * log2(e)
};

struct StageDesc {
    int n_rows;                // -1: no more work
    int work;
    int last;                  // last stage of this split
    int pad;
    uint8_t mask[kAttRows];
};

template <typename T, int D, int G>
struct AttSmem {
    T k[kAttStages][kAttRows][D];
    T v[kAttStages][kAttRows][D];
    float red[kAttWarps / 2][G][D];
    float sw[kAttWarps][G][kAttRowsPerWarp];   // scores, per warp
    float pw[kAttWarps][kAttRowsPerWarp][4];   // probabilities [row][head], per warp
    float cm[kAttWarps][G], cl[kAttWarps][G];
    int scan[kAttWarps + 1];
    StageDesc desc[kAttStages];
    uint64_t bar[kAttStages];
    int work_split, last_flag;
    int prefix[1];                              // [groups + 1], extends past the struct
};

__device__ __forceinline__ void split_shape(int n_items, int& per, int& splits) {
    per = max(kItemsPerSplitMin, (n_items + kSplitMax - 1) / kSplitMax);
    splits = n_items > 0 ? (n_items + per - 1) / per : 0;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kAttThreads, 2) attend_kernel(AttendArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    using Smem = AttSmem<T, D, G>;
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    constexpr int VEC = Elem<T>::kVec;       // elements per 16-byte row load (QK layout)
    constexpr int LPR = D / VEC;             // lanes per row
    constexpr int RPW = 32 / LPR;            // rows per load
    constexpr int U = kAttRowsPerWarp / RPW; // loads per lane per stage
    constexpr int NV = U * G;                // partial dots per lane
    constexpr int VD = D / 32;               // PV: dims per lane
    static_assert(G * kAttRowsPerWarp <= 32, "one lane per (head, row) in the softmax");
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int sub = lane / LPR, li = lane % LPR;

    // ---- split table: prefix[g] = first work id of group g
    {
        int* pre = sm.prefix;
        int carry = 0;
        for (int base = 0; base < a.groups; base += kAttThreads) {
            const int g = base + tid;
            int per, sp = 0;
            if (g < a.groups) split_shape(a.n_items[g], per, sp);
            int tot;
            const int x = block_exclusive_scan<kAttWarps>(sp, sm.scan, &tot);
            if (g < a.groups) pre[g] = carry + x;
            carry += tot;
        }
        if (tid == 0) pre[a.groups] = carry;
        if (tid == 0) {
            for (int i = 0; i < kAttStages; ++i) mbar_init(&sm.bar[i], 1);
            fence_mbar_init();
        }
        __syncthreads();
    }
    const int total_work = sm.prefix[a.groups];
    auto group_of = [&](int work) {   // last g with prefix[g] <= work
        int lo = 0, hi = a.groups - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sm.prefix[mid] <= work) lo = mid; else hi = mid - 1;
        }
        return lo;
    };

    // ---- producer (thread 0): fills stages in work order, packing whole items
    int pw_work = blockIdx.x, p_item = 0, p_end = 0, p_group = 0;
    auto producer_start = [&]() {
        if (pw_work < total_work) {
            p_group = group_of(pw_work);
            const int split = pw_work - sm.prefix[p_group];
            int per, sp;
            split_shape(a.n_items[p_group], per, sp);
            p_item = split * per;
            p_end = min(a.n_items[p_group], p_item + per);
        }
    };
    auto fill = [&](int slot) {
        StageDesc& d = sm.desc[slot];
        if (pw_work >= total_work) {
            d.n_rows = -1;
            mbar_arrive(&sm.bar[slot]);
            return;
        }
        const int2* it = a.items + static_cast<int64_t>(p_group) * a.item_cap;
        int rows = 0, i = p_item;
        while (i < p_end) {
            const int c = it[i].y & 0xffff;
            if (c < 1 || c > kAttRows) {   // never produced by the plans; skip it
                raise_status(ZHA_ERR_INVALID_ARG);
                if (rows == 0) { p_item = ++i; continue; }
                break;
            }
            if (rows + c > kAttRows) break;
            const uint32_t m = static_cast<uint32_t>(it[i].y) >> 16;
            for (int r = 0; r < c; ++r) d.mask[rows + r] = static_cast<uint8_t>(m);
            rows += c;
            ++i;
        }
        d.n_rows = rows;
        d.work = pw_work;
        d.last = i == p_end;
        mbar_arrive_expect_tx(&sm.bar[slot], static_cast<uint32_t>(rows * D * sizeof(T) * 2));
        const int s = p_group / a.Hkv, kv = p_group % a.Hkv;
        const int64_t kvbase = (static_cast<int64_t>(s) * a.Hkv + kv) * a.N_cap;
        const T* Kb = static_cast<const T*>(a.K) + kvbase * D;
        const T* Vb = static_cast<const T*>(a.V) + kvbase * D;
        int r = 0;
        for (int j = p_item; j < i; ++j) {
            const int64_t st = it[j].x;
            const int c = it[j].y & 0xffff;
            if (c < 1 || c > kAttRows) continue;
            const uint32_t bytes = static_cast<uint32_t>(c * D * sizeof(T));
            bulk_g2s(&sm.k[slot][r][0], Kb + st * D, bytes, &sm.bar[slot]);
            bulk_g2s(&sm.v[slot][r][0], Vb + st * D, bytes, &sm.bar[slot]);
            r += c;
        }
        p_item = i;
        if (i == p_end) {
            pw_work += gridDim.x;
            producer_start();
        }
    };
    if (tid == 0) {
        producer_start();
        for (int sl = 0; sl < kAttStages; ++sl) fill(sl);
    }

    // ---- consumer state (every warp)
    float qv[G][VEC];
    float m_run = -INFINITY, l_run = 0.f;      // for head (lane / 8) of this lane
    float acc[G][VD];
    int cur_work = -1;

    int it = 0;
    bool timed_out = false;
    for (;; ++it) {
        const int slot = it % kAttStages;
        const uint32_t parity = (it / kAttStages) & 1;
        const bool ok = mbar_wait_bounded(&sm.bar[slot], parity);
        if (__syncthreads_or(!ok)) {
            timed_out = true;
            break;
        }
        const int n_rows = sm.desc[slot].n_rows;
        if (n_rows < 0) break;
        const int work = sm.desc[slot].work;
        if (work != cur_work) {   // a new split: load q of its group, reset the state
            cur_work = work;
            const int g = group_of(work);
            const int s = g / a.Hkv, kv = g % a.Hkv;
            const T* qp = static_cast<const T*>(a.Q) +
                          ((static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G) * D;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x[VEC];
                Elem<T>::load16(qp + h * D + li * VEC, x);
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
        const int r0 = w * kAttRowsPerWarp;
        if (r0 < n_rows) {
            // QK: lane (sub, li) covers rows r0 + u*RPW + sub, dims [li*VEC, li*VEC+VEC)
            float v[NV];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * RPW + sub;
                float x[VEC];
                if (r < n_rows) {
                    Elem<T>::load16(&sm.k[slot][r][li * VEC], x);
                } else {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) x[e] = 0.f;
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float d = 0.f;
#pragma unroll
                    for (int e = 0; e < VEC; ++e) d = fmaf(qv[h][e], x[e], d);
                    v[h * U + u] = d;
                }
            }
            // transpose-reduce over the LPR lanes of a row group
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
                            const float send = upper ? v[i] : v[i + half];
                            const float keep = upper ? v[i + half] : v[i];
                            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                        }
                    }
                } else {
                    v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
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
                        sm.sw[w][h][u * RPW + sub] = v[k];
                    }
                }
            }
            __syncwarp();
            // online softmax: lane -> (head hh = lane / 8, row rr = lane % 8)
            const int hh = lane / kAttRowsPerWarp, rr = lane % kAttRowsPerWarp;
            const int row = r0 + rr;
            const bool valid = hh < G && row < n_rows && ((sm.desc[slot].mask[row] >> hh) & 1);
            const float sv = valid ? sm.sw[w][hh < G ? hh : 0][rr] : -INFINITY;
            float mx = sv;
#pragma unroll
            for (int o = 1; o < kAttRowsPerWarp; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float mn = fmaxf(m_run, mx);
            const float alpha = mn == -INFINITY ? 1.f : exp2f(m_run - mn);
            const float pr = valid ? exp2f(sv - mn) : 0.f;
            float ps = pr;
#pragma unroll
            for (int o = 1; o < kAttRowsPerWarp; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l_run = l_run * alpha + ps;
            m_run = mn;
            if (hh < G) sm.pw[w][rr][hh] = pr;
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
                if (r0 + r < n_rows) {
                    float vv[VD];
                    load_n<T, VD>(&sm.v[slot][r0 + r][lane * VD], vv);
                    const float4 p4 = *reinterpret_cast<const float4*>(&sm.pw[w][r][0]);
                    const float pp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) acc[h][e] = fmaf(pp[h], vv[e], acc[h][e]);
                }
            }
        }
        if (sm.desc[slot].last) {
            // ---- combine the warps' states into one partial per head
            const int g = group_of(work);
            if (lane % kAttRowsPerWarp == 0 && lane / kAttRowsPerWarp < G) {
                sm.cm[w][lane / kAttRowsPerWarp] = m_run;
                sm.cl[w][lane / kAttRowsPerWarp] = l_run;
            }
            __syncthreads();
            float f[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float M = -INFINITY;
                for (int ww = 0; ww < kAttWarps; ++ww) M = fmaxf(M, sm.cm[ww][h]);
                f[h] = M == -INFINITY ? 0.f : exp2f(sm.cm[w][h] - M);
#pragma unroll
                for (int e = 0; e < VD; ++e) acc[h][e] *= f[h];
            }
#pragma unroll
            for (int half = kAttWarps / 2; half >= 1; half >>= 1) {
                if (w >= half && w < 2 * half)
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) sm.red[w - half][h][lane * VD + e] = acc[h][e];
                __syncthreads();
                if (w < half)
#pragma unroll
                    for (int h = 0; h < G; ++h)
#pragma unroll
                        for (int e = 0; e < VD; ++e) acc[h][e] += sm.red[w][h][lane * VD + e];
                __syncthreads();
            }
            const int split = work - sm.prefix[g];
            if (w == 0) {
                const int64_t pbase = (static_cast<int64_t>(g) * kSplitMax + split) * G;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float M = -INFINITY, Lsum = 0.f;
                    for (int ww = 0; ww < kAttWarps; ++ww) M = fmaxf(M, sm.cm[ww][h]);
                    if (M != -INFINITY)
                        for (int ww = 0; ww < kAttWarps; ++ww) Lsum += sm.cl[ww][h] * exp2f(sm.cm[ww][h] - M);
                    if (lane == 0) a.part_ml[pbase + h] = make_float2(M, Lsum);
#pragma unroll
                    for (int e = 0; e < VD; ++e) a.part_acc[(pbase + h) * D + lane * VD + e] = acc[h][e];
                }
                __threadfence();
            }
            __syncthreads();
            if (tid == 0) {
                int per, sp;
                split_shape(a.n_items[g], per, sp);
                const uint32_t done = atomicAdd(&a.counters[g], 1u);
                sm.last_flag = done == static_cast<uint32_t>(sp - 1);
                sm.work_split = sp;
            }
            __syncthreads();
            if (sm.last_flag) {
                // ---- this CTA closes the group: merge its splits into O
                __threadfence();
                const int sp = sm.work_split;
                const int s = g / a.Hkv, kv = g % a.Hkv;
                for (int x = tid; x < G * D; x += kAttThreads) {
                    const int h = x / D, e = x % D;
                    const int64_t pb = static_cast<int64_t>(g) * kSplitMax * G;
                    float M = -INFINITY;
                    for (int k = 0; k < sp; ++k) M = fmaxf(M, __ldcg(&a.part_ml[pb + k * G + h]).x);
                    float Ls = 0.f, Os = 0.f;
                    if (M != -INFINITY) {
                        for (int k = 0; k < sp; ++k) {
                            const float2 ml = __ldcg(&a.part_ml[pb + k * G + h]);
                            const float f2 = exp2f(ml.x - M);
                            Ls += ml.y * f2;
                            Os += __ldcg(&a.part_acc[(pb + k * G + h) * D + e]) * f2;
                        }
                    }
                    const int64_t orow = (static_cast<int64_t>(s) * a.n_q + (a.n_q - 1)) * a.Hq + kv * G + h;
                    a.O[orow * D + e] = Ls > 0.f ? Os / Ls : 0.f;
                }
                if (tid == 0) a.counters[g] = 0u;
            }
        }
        __syncthreads();   // every warp is done with this slot
        if (tid == 0) fill(slot);
    }
    // Leaving after a timeout: give the copies still in flight a bounded time to
    // land before the CTA's shared memory is released.
    if (timed_out && tid == 0) {
        raise_status(ZHA_ERR_TIMEOUT);
        for (int k = 0; k < kAttStages; ++k)
            mbar_wait_bounded(&sm.bar[(it + k) % kAttStages], ((it + k) / kAttStages) & 1);
    }
}

}  // namespace zha
