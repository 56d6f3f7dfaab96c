/*
 * zha.h -- C ABI of the tree-indexed sparse attention library for NVIDIA B200
 * (sm_100a).
 *
 * The library computes the data-parallel hot path of Zyphra Hierarchical
 * Attention (ZHA) as described on two pages, cited below as
 *   [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured Indexer"
 *   [EoQ] "Zyphra Hierarchical Attention: The End of Quadratic Attention?"
 * The path has three steps: build a tree of recursively compressed key
 * summaries over a KV cache ([HTI] Methodology / Tree Construction), route
 * each query top-down through it with top-p selection at every level ([HTI]
 * Methodology / Routing, m_l(q)), and run exact softmax attention over the
 * selected keys plus the sink token and the current chunk ([HTI] Routing,
 * I(q) and o(q)).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers named K, V, Q, O, N, tree, ws, sel, sel_count, k_new, v_new,
 *   Qref are DEVICE pointers owned by the caller.  `cfg` is a HOST pointer.
 *   The library allocates no device memory: every call works inside the
 *   buffers it is given, on the caller's `stream`, asynchronously.
 * - Layouts (row-major, innermost last):
 *     K, V   [batch][Hkv][N_cap][d]     dtype = cfg->dtype
 *     Q, O   [batch][n_q][Hq][d]        Q in cfg->dtype, O always fp32
 *     Qref   [Hkv][levels][R][d] fp32   levels >= zha_levels_cap(cfg)
 *     N      [batch] int32              keys held in the cache per sequence
 *     sel    [batch][n_q][Hq][sel_cap] int32, sel_count [batch][n_q][Hq] int32
 *   Query head h reads KV head h / (Hq/Hkv) (grouped-query attention).
 * - Every function returns a zha_status.  Host-side checks (bad arguments,
 *   unsupported shapes, a workspace that is too small) return at once and
 *   launch nothing.  Errors found on the device (a full cache, a selection
 *   larger than sel_cap, a bounded wait that ran out) set bits of a sticky
 *   device status word instead; zha_get_status() reads it.  zha_last_error()
 *   returns the message of the calling thread's last failed call.
 * - Device code never traps, asserts or waits without a bound.
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *zha_stream_t;

#define ZHA_MAX_LEVELS 16

typedef enum {
    ZHA_OK = 0,
    ZHA_ERR_INVALID_ARG = 1,  /* null pointer, bad size or inconsistent config       */
    ZHA_ERR_UNSUPPORTED = 2,  /* valid but not built: d not in {64,128}, R > 16, ...   */
    ZHA_ERR_CAPACITY = 3,     /* device: cache full (N == N_cap) or sel_cap exceeded   */
    ZHA_ERR_CUDA = 4,         /* a CUDA runtime call failed (message in last_error)    */
    ZHA_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up (the call returned)    */
    ZHA_ERR_WORKSPACE = 6     /* ws_bytes smaller than zha_workspace_bytes()           */
} zha_status;

typedef enum { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;

/*
 * Geometry and precision.  B = leaf block (keys summarised by one level-1
 * node), b = branching factor (children per node above level 1).  The tree
 * over N keys has n_1 = floor(N/B) leaf nodes (complete blocks only) and
 * n_{l+1} = ceil(n_l / b); its depth is the first level with n_L <= b, or
 * exactly L_fixed levels when L_fixed > 0 (the pages' C4-L6 style).  p[l-1]
 * is the top-p threshold of level l ([HTI] Routing); p >= 1 keeps every
 * candidate.  scale = 0 means 1/sqrt(d).
 */
typedef struct zha_config {
    int32_t d;        /* head dim: 64 or 128                                  */
    int32_t Hq;       /* query heads                                          */
    int32_t Hkv;      /* KV heads; Hq/Hkv in {1, 2, 4}                        */
    int32_t B;        /* leaf block, 1..256 (chunked prefill: 64)             */
    int32_t b;        /* branching factor, 2..32                              */
    int32_t R;        /* reference queries (planes) per node, 1..16           */
    int32_t dtype;    /* zha_dtype of K, V, Q, k_new, v_new                   */
    int32_t batch;    /* sequences                                            */
    int64_t N_cap;    /* rows allocated per (sequence, KV head) in K and V    */
    int32_t L_fixed;  /* 0 = depth rule, else the fixed number of levels      */
    float scale;      /* softmax scale; 0 = 1/sqrt(d)                         */
    float p[ZHA_MAX_LEVELS];
    int32_t vsum;     /* 1: value summaries (decode, R = 1), see below        */
} zha_config;

/*
 * Value summaries (vsum = 1; [HTI] Future Directions (4): pruned subtrees
 * contribute coarse attention outputs).  Every node also stores vhat, the
 * values pooled with the weights that pool its khat (a leaf: softmax(scale
 * qhat.K) V; above: the children's vhat with the children's weights), and
 * decoding adds every node the top-p cut drops as one pseudo-key: log-mass =
 * its routing score s, value = its vhat.  Keys of I(q) that also lie under a
 * dropped node (the sink, a current chunk inside the tree) count in both
 * terms.  zha_build and zha_extend then need V; R must be 1; chunked prefill
 * (n_q > 1) is refused.  vsum = 0 leaves every call as without it.
 */

/* Levels the tree can reach for any N <= N_cap (Qref must hold this many). */
int zha_levels_cap(const zha_config *cfg, int32_t *levels);

/* Bytes of the tree buffer for cfg (summaries of every level up to N_cap,
 * the reference queries, per-sequence counters). */
int zha_tree_bytes(const zha_config *cfg, size_t *bytes);

/* Where level `level` (1 = leaf blocks) lives inside the tree buffer: byte
 * offsets of its khat [batch][Hkv][nodes_cap][R][d] fp32 and bhat
 * [batch][Hkv][nodes_cap][R] fp32 arrays, and nodes_cap.  For inspection. */
int zha_tree_level(const zha_config *cfg, int32_t level, size_t *khat_offset, size_t *bhat_offset,
                   int64_t *nodes_cap);
/* With vsum = 1: byte offset of level `level`'s vhat [batch][Hkv][nodes_cap][d] fp32.
 * ZHA_ERR_INVALID_ARG when vsum = 0. */
int zha_tree_level_v(const zha_config *cfg, int32_t level, size_t *vhat_offset);

/* Byte offset of the per-sequence count of indexed keys, int32 [batch]. */
int zha_tree_count_offset(const zha_config *cfg, size_t *offset);

/* Bytes of the workspace that zha_route/zha_attend/zha_decode/zha_dense need
 * for n_q queries per sequence (decode: n_q = 1; a chunked prefill: n_q > 1,
 * which takes bf16 K/V/Q, leaf blocks of B = 64 and at most 262144 leaf blocks,
 * else ZHA_ERR_UNSUPPORTED).  The workspace must be zeroed once after allocation
 * (zha_workspace_init); calls leave it reusable by any later call whose own
 * size it covers, decode and chunks of any length alike, in any order. */
int zha_workspace_bytes(const zha_config *cfg, int32_t n_q, size_t *bytes);
int zha_workspace_init(const zha_config *cfg, void *ws, size_t ws_bytes, zha_stream_t stream);

/* Accounting left in the workspace by the last calls, for measuring the bytes
 * the path touches: byte offsets of int32 rows[batch*Hkv] (keys gathered per
 * (sequence, KV head) by the last zha_attend / zha_dense plan; with n_q > 1 the
 * number of 64-key blocks the tensor-core attention loaded, each for up to 128
 * query rows), int32 cand[batch][n_q][Hq] (tree nodes scored over all levels
 * for each query head by the last zha_route) and int32 scanned[batch*Hkv]
 * (decode: the distinct tree nodes the last zha_route read per (sequence, KV
 * head), over the query heads that share the KV head; 0 when the route could
 * not count them, for a cache too large for its on-chip bitmaps; with n_q > 1
 * the offset of cand again, each row reading its own candidates). */
int zha_workspace_stats(const zha_config *cfg, int32_t n_q, size_t *rows_offset, size_t *cand_offset,
                        size_t *scanned_offset);

/* Which attention kernel zha_attend (and zha_decode, zha_attend_noalloc) runs for
 * cfg and n_q: *kind = 0 for the CUDA-core decode kernel, 1 for the tensor-core
 * decode kernel (bf16, d = 128, B a multiple of 64, when its shared memory fits
 * the current device), 2 for the tensor-core prefill kernel (n_q > 1).  Reads the
 * current device's limits; launches nothing. */
int zha_attend_kernel(const zha_config *cfg, int32_t n_q, int32_t *kind);

/*
 * zha_build -- build the whole tree over keys [0, N[s]) of every sequence s.
 * [HTI] Tree Construction: each complete block of B keys gets, for its
 * reference query qhat, the tangent of F_C(q) = LSE_j(q.k_j * scale) at qhat:
 * khat = softmax(scale qhat.K) K and bhat = F_C(qhat) - scale qhat.khat.
 * Upper levels are "constructed recursively from their children's
 * summaries": each child is a pseudo-key of log-mass scale q.khat_c + bhat_c,
 * and the node is the tangent of their LSE at the level's reference query.
 * Qref is copied into the tree.  N is read on the device.  V (the value cache,
 * laid out as K) is read only with vsum = 1, and may then not be NULL.
 */
int zha_build(const zha_config *cfg, const void *K, const void *V, const float *Qref, const int32_t *N,
              void *tree, zha_stream_t stream);

/*
 * zha_extend -- grow the tree to index keys [0, N[s]) of every sequence s whose
 * rows the caller has already written into K (for instance a prefill chunk):
 * the new complete leaf blocks are summarised, then their ancestors and any new
 * level ([EoQ] "the tree is built on the fly as the context grows").  The
 * result is bitwise equal to zha_build at N.  N[s] below the tree's current
 * count, or above N_cap, sets ZHA_ERR_INVALID_ARG on the device and leaves
 * that sequence's count unchanged.  V as for zha_build.
 */
int zha_extend(const zha_config *cfg, const void *K, const void *V, const int32_t *N, void *tree,
               zha_stream_t stream);

/*
 * zha_append -- decode-time growth ([EoQ] "the tree is built on the fly as the
 * context grows").  For every sequence s, writes k_new[s][h], v_new[s][h]
 * (layout [batch][Hkv][d]) at row N[s] of K and V, increments N[s], and, when
 * that completes a leaf block, summarises the block and recomputes its
 * ancestors (adding a level when the top outgrows b).  The result is bitwise
 * equal to zha_build at the new N.  A full cache (N == N_cap) sets
 * ZHA_ERR_CAPACITY in the device status and leaves that sequence unchanged.
 */
int zha_append(const zha_config *cfg, void *K, void *V, const void *k_new, const void *v_new,
               int32_t *N, void *tree, zha_stream_t stream);

/*
 * zha_route -- top-down top-p routing of decode queries (n_q = 1, query at
 * position t = N[s]-1).  [HTI] Routing: level L's candidates are all its
 * nodes; each candidate scores s = scale q.khat + bhat; the kept set is the
 * smallest prefix, in descending score order (ties to the lower node id), whose
 * normalised mass reaches p_l; the children of kept nodes are the next
 * level's candidates.  Writes the kept level-1 block ids of every (sequence,
 * query head), ascending, to sel (capacity sel_cap per row) and their count to
 * sel_count.  A count above sel_cap sets ZHA_ERR_CAPACITY on the device (the
 * first sel_cap ids are written).  It also leaves in ws the gather plan of
 * zha_attend for these selections (see zha_attend with sel == NULL).
 */
/*
 * zha_route with n_q > 1 -- a chunked prefill.  N[s] counts the keys in the
 * cache including the chunk's n_q keys, which the caller has written at rows
 * [N[s] - n_q, N[s]) of K and V; the tree must index exactly the N[s] - n_q keys
 * before the chunk (else ZHA_ERR_INVALID_ARG on the device and empty
 * selections).  Query i of the chunk sits at t = N[s] - n_q + i.  Each (query,
 * query head) is routed as above, independently.  No gather plan is left in ws.
 */
int zha_route(const zha_config *cfg, const void *tree, const void *Q, int32_t n_q, const int32_t *N,
              int32_t *sel, int32_t *sel_count, int32_t sel_cap, void *ws, size_t ws_bytes,
              zha_stream_t stream);

/*
 * zha_attend -- exact softmax attention over I(q) = {0} u (keys of the listed
 * level-1 blocks) u C_cur(t) ([HTI] Routing, I(q) and o(q) = Attn(q, K_I, V_I);
 * the first token is the sink, [EoQ]).  C_cur(t) = [min(floor(t/B), n_1)*B, t]
 * with n_1 the number of leaf blocks in the tree.  n_q = 1 (decode, t =
 * N[s]-1).  The blocks of the query heads that share a KV head are loaded once.
 * O is fp32 [batch][n_q][Hq][d].  tree is read only for n_1.  With sel == NULL
 * the gather plan that the last zha_route on this workspace left is used
 * (sel_count and sel_cap are then ignored).
 */
/*
 * zha_attend with n_q > 1 -- the chunked prefill's attention, on the tensor
 * cores.  Same index set with C_cur(t) = [n_1*B, t], the causal tail (n_1 = the
 * tree's leaf blocks, the tree indexing the N[s] - n_q keys before the chunk).
 * sel and sel_count are required; each row's list must be ascending and below
 * n_1 (else ZHA_ERR_INVALID_ARG on the device, and the valid prefix is used).
 * The softmax weights are rounded to bf16 for the P V product (their sum is
 * taken over the rounded values), so an output moves by at most 2^-8 max|v|
 * against exact attention over the same set.  Deterministic: the same inputs
 * give bitwise the same outputs.
 */
int zha_attend(const zha_config *cfg, const void *K, const void *V, const void *tree,
               const void *Q, int32_t n_q, const int32_t *N, const int32_t *sel,
               const int32_t *sel_count, int32_t sel_cap, float *O, void *ws, size_t ws_bytes,
               zha_stream_t stream);

/*
 * zha_attend_noalloc -- zha_attend for callers that cannot allocate device
 * memory and so cannot hand in a workspace: code embedded in a host framework
 * that owns every device allocation and exposes no allocator to it, or a
 * serving path that is not allowed to call cudaMalloc (it can synchronise the
 * device and fragment a pre-reserved pool).  The pages describe no counterpart;
 * it is a convenience of this library.
 *
 * Decode only: n_q must be 1 (a chunked prefill, n_q > 1, is refused with
 * ZHA_ERR_UNSUPPORTED before anything runs), and vsum = 1 is refused likewise.
 * Otherwise arguments, layouts and results are those of zha_attend with n_q = 1
 * (sel must not be NULL), bit for bit; the caller still owns K, V, tree, Q, N,
 * sel, sel_count and O.  The
 * scratch is one static device array of 16 MiB inside the library, present on
 * every GPU that loads the library until the process exits.  A configuration
 * whose scratch (zha_workspace_bytes) exceeds 16 MiB is refused with
 * ZHA_ERR_WORKSPACE before anything runs.  The call allocates nothing.
 * - The first call on a device (in each CUDA context of that device) looks
 *   the array's device address up with cudaGetSymbolAddress; make that first
 *   call before any stream capture.
 * - All calls on a device share the array and it keeps the last call's
 *   contents: calls that may overlap on the GPU (two streams, or two host
 *   threads) race on it and must be serialised by the caller.
 */
int zha_attend_noalloc(const zha_config *cfg, const void *K, const void *V, const void *tree,
                       const void *Q, int32_t n_q, const int32_t *N, const int32_t *sel,
                       const int32_t *sel_count, int32_t sel_cap, float *O, zha_stream_t stream);

/* zha_decode -- one decode step: zha_append, then zha_route and zha_attend of
 * the query q [batch][1][Hq][d] at its own position (t = new N - 1).  The
 * selection goes to the workspace. */
int zha_decode(const zha_config *cfg, void *K, void *V, void *tree, const void *q,
               const void *k_new, const void *v_new, int32_t *N, float *O, void *ws,
               size_t ws_bytes, zha_stream_t stream);

/* zha_dense -- the in-library dense baseline: attention of q [batch][1][Hq][d]
 * over every key [0, N[s]), with the same loader as zha_attend.  With n_q > 1,
 * causal dense attention of the chunk's queries (query i over [0, N[s] - n_q +
 * i]) on the tensor-core kernel of zha_attend's prefill; tree is not needed. */
int zha_dense(const zha_config *cfg, const void *K, const void *V, const void *Q, int32_t n_q,
              const int32_t *N, float *O, void *ws, size_t ws_bytes, zha_stream_t stream);

/* Reads (and if clear != 0 resets) the sticky device status of the current
 * device: bit (1 << code) for each zha_status code raised on the device since
 * the last clear.  Synchronises `stream`. */
int zha_get_status(int32_t *status_bits, int32_t clear, zha_stream_t stream);

/* Bound, in nanoseconds, of the tensor-core decode attention's waits on the
 * progress of its other warps (default 2e9; it applies to kernels launched
 * after the call, on every device, and returns the previous bound in
 * *previous when that is not NULL).  A control for testing the failure path:
 * with 0, a wait that is not already satisfied gives up at once.  A wait that
 * gives up raises ZHA_ERR_TIMEOUT in the device status; the CTA then stops
 * work, lets the copies and MMAs it issued itself complete (those waits keep
 * the 2 s bound), frees its tensor memory and returns, so the call always
 * ends.  The output of that call is undefined, and so are the merge counters
 * it leaves in the workspace: re-initialise the workspace (zha_workspace_init)
 * before reusing it.  The other kernels' waits keep the 2 s bound. */
int zha_set_wait_limit(uint64_t ns, uint64_t *previous);

/* Message of the calling thread's last failed call ("" if none). */
const char *zha_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* ZHA_H */
