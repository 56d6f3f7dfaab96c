// zha_score_tc.cuh -- the scores of every upper-level tree node for a chunk of
// prefill queries, as dense tensor-core products (sm_100a tcgen05).
//
// Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
// Indexer", Methodology / Routing: a candidate node scores its tangent estimate
// s = scale * q.khat + bhat.  In a chunked prefill every query row of one
// (sequence, KV head) is routed through the same tree, and above the leaf blocks
// the levels are small (at 256K: 256 + 16 nodes) while the rows are many (4096
// queries x 4 heads): most rows score most upper nodes, so those scores are one
// dense contraction, Q [rows x d] . Khat^T [d x nodes].  This kernel computes it
// for all upper nodes of 128-row tiles; the router then reads a row's scores at
// those levels instead of scanning the children, and scans only the leaf level
// (whose candidates differ from row to row).
//
// Precision: the summaries are fp32 and the tensor cores take bf16 operands.
// Each fp32 khat is split exactly into three bf16 parts,
//   hi = bf16(x), mid = bf16(x - hi), lo = bf16(x - hi - mid),  x = hi + mid + lo
// (each residual is exact in fp32 and the last fits bf16's 8 significant bits),
// and q is bf16 already, so q.khat = q.hi + q.mid + q.lo is a sum of exact
// products accumulated in fp32 -- fp32-grade scores, as the CUDA-core scan gives.
//
// The summaries' split is the same for every query tile, so split_upper_kernel
// does it once per (sequence, KV head): 64 nodes at a time, the three bf16 parts
// go to global memory already in the 128-byte-swizzled K-major layout the tensor
// cores read, with the 64 biases beside them.  score_upper_kernel then runs one
// CTA of 256 threads per (sequence, KV head, 128-row tile): the Q tile goes to
// shared memory once (swizzled, K-major), and per 64-node chunk one bulk copy
// brings the operand tiles, thread 0 issues the 3 x d/16 MMAs (M = 128 rows,
// N = 64 nodes, fp32 accumulators in TMEM), and the rows' accumulators are read
// back, biased and written (warps w and w + 4 share TMEM lanes 32 (w mod 4) ..
// +31, i.e. the same rows, and take 32 columns each).  Two CTAs fit on an SM.
// Waits are bounded (a timeout raises ZHA_ERR_TIMEOUT and the CTA stops issuing).
#pragma once

#include <cuda_bf16.h>

#include "zha_common.cuh"
#include "zha_umma.cuh"

namespace zha {

constexpr int kSUThreads = 256;   // rows = TMEM lanes: warps w and w + 4 both hold lanes 32 (w mod 4) ..
constexpr int kSUNodes = 64;      // nodes per MMA (N)
constexpr int kSUTileRows = 128;  // M
constexpr int kSUMaxCols = 2048;  // upper nodes (over all upper levels) this path takes
constexpr int kSUStage = 65;      // floats per row of the staged scores (64, padded against bank conflicts)

struct SUArgs {
    const uint16_t* Q;        // [batch][n_q][Hq][D] bf16
    TreeDev tree;
    const int32_t* N;         // [batch], keys including the chunk
    float* up;                // [slices][R][ucap] scores of upper nodes: column up_off[l-1] + node for level l
    unsigned char* split;     // [slices][chunk_cap] operand tiles of 64 nodes (SULayout::kBBytes each)
    float* bias;              // [slices][chunk_cap][64]
    int64_t ucap, N_cap;
    int up_off[kMaxLevels];   // column offset of level l (index l - 1), l >= 2
    int chunk_cap;
    int n_q, Hq, Hkv, G, B, b, L_fixed, R, slices, tiles;
    float scale;
};

template <int D>
struct SULayout {
    static constexpr int kH = D / 64;                                  // 64-element spans
    static constexpr uint32_t kQBytes = kH * kSUTileRows * 128;        // Q tile
    static constexpr uint32_t kPartBytes = kH * kSUNodes * 128;        // one bf16 part of 64 nodes
    static constexpr uint32_t kBBytes = 3 * kPartBytes;                // hi, mid, lo
    static constexpr uint32_t kStageBytes = kSUTileRows * kSUStage * 4; // the scores staged for the write
    static constexpr uint32_t kBArea = ((kBBytes > kStageBytes ? kBBytes : kStageBytes) + 1023u) & ~1023u;
    static constexpr uint32_t kOffB = kQBytes;                         // the operand tiles, then the stage
    static constexpr uint32_t kOffBias = kOffB + kBArea;               // 64 biases
    static constexpr uint32_t kOffCtl = kOffBias + kSUNodes * 4;
    static constexpr size_t kSmem = kOffCtl + 64 + 1024;               // + control, alignment slack
};

struct SUCtl {
    uint64_t mma_done;        // MMA -> all: a chunk's products are in TMEM
    uint64_t full;            // bulk copy -> all: a chunk's operand tiles and biases landed
    uint32_t tmem;
    int abort;
};

// Splits 8 fp32 values into their three bf16 parts, as 3 x 16 bytes.
__device__ __forceinline__ void split3(const float* x, uint4* hi, uint4* mid, uint4* lo) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * k]), h1 = __float2bfloat16_rn(x[2 * k + 1]);
        const float r0 = x[2 * k] - __bfloat162float(h0), r1 = x[2 * k + 1] - __bfloat162float(h1);
        __nv_bfloat16 m0 = __float2bfloat16_rn(r0), m1 = __float2bfloat16_rn(r1);
        __nv_bfloat16 l0 = __float2bfloat16_rn(r0 - __bfloat162float(m0)), l1 = __float2bfloat16_rn(r1 - __bfloat162float(m1));
        h[k] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        m[k] = static_cast<uint32_t>(__bfloat16_as_ushort(m0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(m1)) << 16);
        l[k] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
    }
    *hi = make_uint4(h[0], h[1], h[2], h[3]);
    *mid = make_uint4(m[0], m[1], m[2], m[3]);
    *lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// The (level, first node) of chunk c of a tree whose level sizes are n[]: chunks of 64 nodes,
// levels 2, 3, ... in turn.  Returns false past the last chunk.
__device__ __forceinline__ bool su_chunk(const int64_t* n, int L, int c, int* level, int64_t* n0) {
    for (int l = 2; l <= L; ++l) {
        const int k = static_cast<int>((static_cast<uint32_t>(n[l - 1]) + kSUNodes - 1) / kSUNodes);
        if (c < k) {
            *level = l;
            *n0 = static_cast<int64_t>(c) * kSUNodes;
            return true;
        }
        c -= k;
    }
    return false;
}

// One CTA per (sequence, KV head, 64-node chunk): the chunk's summaries split into their
// three bf16 parts, in the swizzled operand layout, and its biases.
template <int D>
__global__ void __launch_bounds__(256) split_upper_kernel(SUArgs a) {
    using Lay = SULayout<D>;
    const int slice = blockIdx.x / a.chunk_cap, c = blockIdx.x % a.chunk_cap;
    const int s = slice / a.Hkv;
    const int64_t N = a.N[s];
    const int64_t Ntree = a.tree.n_tree[s];
    if (N < a.n_q || N > a.N_cap || Ntree != N - a.n_q) return;
    int64_t n[kMaxLevels];
    const int L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
    int l;
    int64_t n0;
    if (L < 2 || !su_chunk(n, L, c, &l, &n0)) return;
    const int cnt = static_cast<int>(min(static_cast<int64_t>(kSUNodes), n[l - 1] - n0));
    const int64_t ncap = a.tree.ncap[l - 1];
    const float* kh = a.tree.khat[l - 1] + static_cast<int64_t>(slice) * ncap * D;
    unsigned char* dstB = a.split + (static_cast<int64_t>(slice) * a.chunk_cap + c) * Lay::kBBytes;
    for (int x = threadIdx.x; x < kSUNodes * (D / 8); x += blockDim.x) {
        const int node = x / (D / 8), cc8 = x % (D / 8);
        float v[8];
        if (node < cnt) {
            const float4* src = reinterpret_cast<const float4*>(kh + (n0 + node) * D + cc8 * 8);
            const float4 u0 = __ldg(src), u1 = __ldg(src + 1);
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
            v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = 0.f;
        }
        uint4 hi, mid, lo;
        split3(v, &hi, &mid, &lo);
        const int half = cc8 >> 3, cc = cc8 & 7;
        const uint32_t off = half * (kSUNodes * 128) + node * 128 + ((cc ^ (node & 7)) << 4);
        *reinterpret_cast<uint4*>(dstB + off) = hi;
        *reinterpret_cast<uint4*>(dstB + Lay::kPartBytes + off) = mid;
        *reinterpret_cast<uint4*>(dstB + 2 * Lay::kPartBytes + off) = lo;
    }
    const float* bh = a.tree.bhat[l - 1] + static_cast<int64_t>(slice) * ncap;
    if (threadIdx.x < kSUNodes)
        a.bias[(static_cast<int64_t>(slice) * a.chunk_cap + c) * kSUNodes + threadIdx.x] =
            static_cast<int>(threadIdx.x) < cnt ? bh[n0 + threadIdx.x] : 0.f;
}

template <int D>
__global__ void __launch_bounds__(kSUThreads, 2) score_upper_kernel(SUArgs a) {
    using Lay = SULayout<D>;
    extern __shared__ __align__(1024) unsigned char su_smem[];
    const uint32_t raw_s = smem_addr(su_smem);
    unsigned char* base = su_smem + (((raw_s + 1023u) & ~1023u) - raw_s);
    unsigned char* sQ = base;
    unsigned char* sB = base + Lay::kOffB;
    float* sBias = reinterpret_cast<float*>(base + Lay::kOffBias);
    SUCtl* ctl = reinterpret_cast<SUCtl*>(base + Lay::kOffCtl);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int slice = blockIdx.x / a.tiles, tile = blockIdx.x % a.tiles;
    const int s = slice / a.Hkv, kv = slice % a.Hkv;
    const int64_t N = a.N[s];
    const int64_t Ntree = a.tree.n_tree[s];
    // the route checks and reports these; here the tile is skipped
    if (N < a.n_q || N > a.N_cap || Ntree != N - a.n_q) return;
    int64_t n[kMaxLevels];
    const int L = tree_levels(Ntree, a.B, a.b, a.L_fixed, n);
    if (L < 2) return;

    if (tid == 0) {
        mbar_init(&ctl->mma_done, 1);
        mbar_init(&ctl->full, 1);
        fence_mbar_init();
        ctl->abort = 0;
    }
    if (warp == 0) {
        umma::tmem_alloc(&ctl->tmem, kSUNodes);
        umma::tmem_relinquish();
    }
    // ---- the tile's Q rows: row r = (query r / G, head r % G of this KV head); 16-byte chunks
    // spread over all threads
    for (int x = tid; x < kSUTileRows * (D / 8); x += kSUThreads) {
        const int row = x / (D / 8), c = x % (D / 8);
        const int r = tile * kSUTileRows + row;
        const bool ok = r < a.R;
        const int64_t grow = (static_cast<int64_t>(s) * a.n_q + (ok ? r / a.G : 0)) * a.Hq + kv * a.G + (ok ? r % a.G : 0);
        const int half = c >> 3, cc = c & 7;
        unsigned char* dst = sQ + half * (kSUTileRows * 128) + row * 128 + ((cc ^ (row & 7)) << 4);
        umma::cp_async16(dst, ok ? static_cast<const void*>(a.Q + grow * D + c * 8) : a.Q, ok);
    }
    umma::cp_async_wait_all();
    umma::fence_proxy_async_smem();
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem;
    const int row = (warp & 3) * 32 + lane;          // the TMEM lane this thread reads
    const int col0 = (warp >> 2) * 32;               // and its 32 of the chunk's 64 columns
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr uint32_t kId = umma::idesc_bf16(kSUTileRows, kSUNodes, false);
    float* stage = reinterpret_cast<float*>(sB);   // 128 rows of scores, once the MMAs read the tiles

    // chunks of 64 nodes of each level l >= 2; chunk c's bulk copy completes phase c of full,
    // its commit phase c of mma_done
    bool inflight = false;   // the MMAs of chunk inflight_c were issued and not yet waited for
    int inflight_c = 0;
    const unsigned char* gB = a.split + static_cast<int64_t>(slice) * a.chunk_cap * Lay::kBBytes;
    const float* gBias = a.bias + static_cast<int64_t>(slice) * a.chunk_cap * kSUNodes;
    int chunk = 0;
    int l;
    int64_t n0;
    for (; !ctl->abort && su_chunk(n, L, chunk, &l, &n0); ++chunk) {
        const int cnt = static_cast<int>(min(static_cast<int64_t>(kSUNodes), n[l - 1] - n0));
        if (tid == 0) {
            mbar_arrive_expect_tx(&ctl->full, Lay::kBBytes + kSUNodes * 4);
            bulk_g2s(sB, gB + static_cast<int64_t>(chunk) * Lay::kBBytes, Lay::kBBytes, &ctl->full);
            bulk_g2s(sBias, gBias + static_cast<int64_t>(chunk) * kSUNodes, kSUNodes * 4, &ctl->full);
        }
        // the copies always land: wait with the long bound, so no copy is left in flight
        const bool landed = mbar_wait_bounded(&ctl->full, static_cast<uint32_t>(chunk) & 1u, kWaitLongNs);
        if (!landed) {
            if (tid == 0) raise_status(ZHA_ERR_TIMEOUT);
            ctl->abort = 1;
        }
        __syncthreads();
        if (ctl->abort) break;
        if (tid == 0) {
            umma::fence_after_sync();
            bool first = true;
#pragma unroll
            for (int part = 0; part < 3; ++part)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = umma::desc_sw128(smem_addr(sQ + (kk >> 2) * (kSUTileRows * 128) + (kk & 3) * 32), 16, 1024);
                    const uint64_t bd = umma::desc_sw128(
                        smem_addr(sB + part * Lay::kPartBytes + (kk >> 2) * (kSUNodes * 128) + (kk & 3) * 32), 16, 1024);
                    umma::mma_bf16(tmem, ad, bd, kId, first ? 0u : 1u);
                    first = false;
                }
            umma::commit(&ctl->mma_done);
        }
        inflight = true;
        inflight_c = chunk;
        // ---- the chunk's 64 scores of every row (this thread: 32 of them) -> global
        bool got = mbar_wait_bounded(&ctl->mma_done, static_cast<uint32_t>(chunk) & 1u);
        got = __all_sync(0xffffffffu, got);   // the TMEM load below is warp-wide
        if (!got) {
            if (lane == 0) raise_status(ZHA_ERR_TIMEOUT);
            ctl->abort = 1;
        } else {
            inflight = false;
            umma::fence_after_sync();
            float v[32];
            umma::tmem_ld32(tmem + col0 + lane_base, v);
            // through shared memory (the consumed operand tiles), so that the global writes
            // below are whole 128-byte row segments
#pragma unroll
            for (int k = 0; k < 32; ++k) stage[row * kSUStage + col0 + k] = fmaf(a.scale, v[k], sBias[col0 + k]);
        }
        umma::fence_before_sync();
        __syncthreads();
        if (!ctl->abort)
            for (int rr = warp; rr < kSUTileRows; rr += kSUThreads / 32) {
                const int rg = tile * kSUTileRows + rr;
                if (rg >= a.R) break;
                float* drow = a.up + (static_cast<int64_t>(slice) * a.R + rg) * a.ucap + a.up_off[l - 1] + n0;
                if (lane < cnt) drow[lane] = stage[rr * kSUStage + lane];
                if (32 + lane < cnt) drow[32 + lane] = stage[rr * kSUStage + 32 + lane];
            }
        __syncthreads();   // the operand tiles, the biases and the TMEM block are free again
    }
    // every MMA issued has completed before the TMEM goes back (after an abort, the last
    // chunk's commit is waited for here)
    if (inflight && tid == 0) mbar_wait_bounded(&ctl->mma_done, static_cast<uint32_t>(inflight_c) & 1u, kWaitLongNs);
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kSUNodes);
    }
}

}  // namespace zha
