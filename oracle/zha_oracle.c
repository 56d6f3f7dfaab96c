/*
 * zha_oracle.c -- the fp64 CPU oracle of tree-indexed sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA path computes.  Only the tests, the package's
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header or constant with the CUDA library.
 *
 * Pages cited (title, then section / equation):
 *   [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured Indexer"
 *   [EoQ] "Zyphra Hierarchical Attention: The End of Quadratic Attention?"
 *
 * Every function works on ONE (sequence, KV head) slice.  Arithmetic is
 * double precision throughout; inputs are fp32 or bf16 values, widened.
 * No blocking, fusion or reordering beyond what the definitions state.
 *
 * Parity: leaf summary, upper-level summary, routing, index set and
 * attention are each pinned by tests (closed forms, brute force, the p = 1
 * dense limit, tangent exactness); so are the value summaries (uniform
 * blocks, a linear map V = K M, the partition of the tree by kept blocks and
 * dropped nodes, exactness when every top node holds one key).  The routing
 * margin (how far a cut lies from p; a test-side construct the pages do not
 * define) and the generators are "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- element access: dtype 0 = fp32, 1 = bf16 (upper 16 bits of an fp32) ---- */
static double elem(const void *base, int dtype, int64_t i) {
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double dot_slice(const double *q, const void *K, int dtype, int64_t row, int d) {
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += q[e] * elem(K, dtype, row * d + e);
    return s;
}

static double dot(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += a[e] * b[e];
    return s;
}

/* log-sum-exp of z[0..n), n >= 1 */
static double lse(const double *z, int64_t n) {
    double m = z[0];
    for (int64_t i = 1; i < n; ++i) if (z[i] > m) m = z[i];
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i) s += exp(z[i] - m);
    return m + log(s);
}

/*
 * Geometry.  n_1 = floor(N/B) complete leaf blocks; n_{l+1} = ceil(n_l / b);
 * L = the first level with n_L <= b, or exactly L_fixed levels when
 * L_fixed > 0 (the pages' "C4-L6"-style geometries fix the depth and let the
 * top level hold many nodes).  [HTI] Tree Construction ("higher-level nodes
 * span C^l keys"), read with a separate leaf size B and fan-out b.
 * Writes n[0..L) (n[l-1] = nodes of level l) and returns L, or -1 when more
 * than max_levels levels would be needed.
 */
int oracle_levels(int64_t N, int B, int b, int L_fixed, int64_t *n, int max_levels) {
    int64_t cur = N / B;
    int L = 1;
    if (max_levels < 1 || L_fixed > max_levels) return -1;
    n[0] = cur;
    while (L_fixed > 0 ? L < L_fixed : cur > b) {
        cur = (cur + b - 1) / b;
        if (L >= max_levels) return -1;
        n[L++] = cur;
    }
    return L;
}

/*
 * Tree build.  Level l occupies nodes [off_l, off_l + n_l) of khat/bhat,
 * off_l = n_1 + ... + n_{l-1}; node storage is khat[node][r][d], bhat[node][r].
 * qref is [L][R][d] (level-major), scale is 1/sqrt(d).
 *
 * Leaf ([HTI] Tree Construction, F_C and the tangent at q-hat_r):
 *   z_i = scale * qhat . k_i over the B keys of the block,
 *   F = LSE(z), w = softmax(z) = exp(z - F), khat = sum_i w_i k_i,
 *   bhat = F - scale * qhat . khat.
 * Upper level ("constructed recursively from their children's summaries"):
 *   each child c is a pseudo-key with log-mass s_c(x) = max_r' (scale x.khat_{c,r'} + bhat_{c,r'});
 *   the node's plane r is the tangent of LSE_c s_c(x) at qhat_{l,r}:
 *   z_c = s_c(qhat), w = softmax(z), khat = sum_c w_c khat_{c,r*(c)}
 *   (r* = the plane attaining the max, lowest r' on ties), bhat = LSE(z) - scale qhat.khat.
 */
void oracle_build_v(const void *K, const void *V, int dtype, int64_t N, int d, int B, int b, int R, int L,
                    const double *qref, double scale, double *khat, double *bhat, double *vhat);

void oracle_build(const void *K, int dtype, int64_t N, int d, int B, int b, int R, int L,
                  const double *qref, double scale, double *khat, double *bhat) {
    oracle_build_v(K, NULL, dtype, N, d, B, b, R, L, qref, scale, khat, bhat, NULL);
}

/*
 * The same build, and, when V and vhat are given, the value summaries ([HTI]
 * Future Directions (4): pruned subtrees contribute coarse attention outputs).
 * Reading: the value summary is pooled with the weights that pool the key
 * summary -- vhat_r = Attn(qhat_r, K_C, V_C) = sum_i w_i v_i at a leaf; at an
 * upper node, sum_c w_c vhat_{c,r*(c)} with the children's weights w_c and best
 * planes r*(c) of khat.  vhat has the layout of khat: [node][R][d].
 */
void oracle_build_v(const void *K, const void *V, int dtype, int64_t N, int d, int B, int b, int R, int L,
                    const double *qref, double scale, double *khat, double *bhat, double *vhat) {
    int64_t n[64];
    if (oracle_levels(N, B, b, L, n, 64) != L) return;
    double *z = (double *)malloc(sizeof(double) * (size_t)(B > b ? B : b));
    int *rs = (int *)malloc(sizeof(int) * (size_t)b);

    /* level 1: leaf blocks of raw keys */
    for (int64_t j = 0; j < n[0]; ++j) {
        for (int r = 0; r < R; ++r) {
            const double *q = qref + (0 * R + r) * d;
            for (int i = 0; i < B; ++i) z[i] = scale * dot_slice(q, K, dtype, j * B + i, d);
            double F = lse(z, B);
            double *kh = khat + (j * R + r) * d;
            for (int e = 0; e < d; ++e) kh[e] = 0.0;
            for (int i = 0; i < B; ++i) {
                double w = exp(z[i] - F);
                for (int e = 0; e < d; ++e) kh[e] += w * elem(K, dtype, (j * B + i) * d + e);
            }
            if (vhat) {
                double *vh = vhat + (j * R + r) * d;
                for (int e = 0; e < d; ++e) vh[e] = 0.0;
                for (int i = 0; i < B; ++i) {
                    double w = exp(z[i] - F);
                    for (int e = 0; e < d; ++e) vh[e] += w * elem(V, dtype, (j * B + i) * d + e);
                }
            }
            bhat[j * R + r] = F - scale * dot(q, kh, d);
        }
    }

    /* levels 2..L from their children */
    int64_t off_child = 0, off = n[0];
    for (int l = 2; l <= L; ++l) {
        int64_t nl = n[l - 1], nc = n[l - 2];
        for (int64_t i = 0; i < nl; ++i) {
            int64_t c0 = i * b, c1 = c0 + b < nc ? c0 + b : nc;
            for (int r = 0; r < R; ++r) {
                const double *q = qref + ((int64_t)(l - 1) * R + r) * d;
                for (int64_t c = c0; c < c1; ++c) {
                    /* The child's estimate is the max over its planes, taken exactly
                     * ([HTI] Tree Construction: max over r of t_r); r*(c) is the plane
                     * that attains it, the lowest one on an exact tie. */
                    double best = -INFINITY;
                    int br = 0;
                    for (int r2 = 0; r2 < R; ++r2) {
                        int64_t node = off_child + c;
                        double t = scale * dot(q, khat + (node * R + r2) * d, d) + bhat[node * R + r2];
                        if (t > best) { best = t; br = r2; }
                    }
                    z[c - c0] = best;
                    rs[c - c0] = br;
                }
                double F = lse(z, c1 - c0);
                double *kh = khat + ((off + i) * R + r) * d;
                for (int e = 0; e < d; ++e) kh[e] = 0.0;
                for (int64_t c = c0; c < c1; ++c) {
                    double w = exp(z[c - c0] - F);
                    const double *kc = khat + ((off_child + c) * R + rs[c - c0]) * d;
                    for (int e = 0; e < d; ++e) kh[e] += w * kc[e];
                }
                if (vhat) {
                    double *vh = vhat + ((off + i) * R + r) * d;
                    for (int e = 0; e < d; ++e) vh[e] = 0.0;
                    for (int64_t c = c0; c < c1; ++c) {
                        double w = exp(z[c - c0] - F);
                        const double *vc = vhat + ((off_child + c) * R + rs[c - c0]) * d;
                        for (int e = 0; e < d; ++e) vh[e] += w * vc[e];
                    }
                }
                bhat[(off + i) * R + r] = F - scale * dot(q, kh, d);
            }
        }
        off_child = off;
        off += nl;
    }
    free(z);
    free(rs);
}

/* ---- routing ---- */
typedef struct { double s; int64_t id; int plane; } scored_t;

/* descending score; ties go to the lower node id */
static int cmp_scored(const void *a, const void *b) {
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

static int cmp_i64(const void *a, const void *b) {
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

/*
 * Top-down routing of one query through a tree of L levels built over N keys
 * ([HTI] Routing, m_l(q); [EoQ] How the tree is built and searched).  Level L's candidates are all its nodes; level l < L's
 * are the children of the nodes kept at l+1.  Each candidate scores
 * s = max_r (scale q.khat_r + bhat_r).  Candidates are ordered by s
 * (descending, ties to the lower id); the kept set is the smallest prefix whose
 * normalised mass sum exp(s_i) / sum_candidates exp(s_j) reaches p_l, and
 * p_l >= 1 keeps every candidate.
 *
 * Outputs: sel[0..count) = kept level-1 block ids, ascending (capacity n_1);
 * per level l (index l-1): n_cand[l-1], n_kept[l-1], margin[l-1] with
 * margin = min(c_m - p, p - c_{m-1}, s_(m) - s_(m+1)): the distance of the
 * cumulative normalised mass from p on both sides of the cut, and the score
 * gap (log-mass units) between the last kept and the first dropped candidate
 * (absent terms = +inf).
 * Returns the count.
 */
int64_t oracle_route2(const double *q, int d, int R, int B, int b, int64_t N, int L,
                      const double *khat, const double *bhat, double scale, const double *p,
                      int64_t *sel, int64_t *n_cand, int64_t *n_kept, double *margin,
                      int64_t *pr_node, int *pr_plane, double *pr_s, int64_t *n_pr);

int64_t oracle_route(const double *q, int d, int R, int B, int b, int64_t N, int L,
                     const double *khat, const double *bhat, double scale, const double *p,
                     int64_t *sel, int64_t *n_cand, int64_t *n_kept, double *margin) {
    return oracle_route2(q, d, R, B, b, N, L, khat, bhat, scale, p, sel, n_cand, n_kept, margin,
                         NULL, NULL, NULL, NULL);
}

/*
 * The same routing, and, when pr_node is given, the pruned nodes: at every level
 * the candidates the cut drops (their subtrees are not searched further), as
 * global node indices (level 1 first, the layout of khat), each with its score
 * s and the plane attaining it (lowest plane on ties).  Kept level-1 blocks and
 * the leaves under pruned nodes partition the tree's blocks.  pr_* need room for
 * every node of the tree; *n_pr gets the count.
 */
int64_t oracle_route2(const double *q, int d, int R, int B, int b, int64_t N, int L,
                      const double *khat, const double *bhat, double scale, const double *p,
                      int64_t *sel, int64_t *n_cand, int64_t *n_kept, double *margin,
                      int64_t *pr_node, int *pr_plane, double *pr_s, int64_t *n_pr) {
    int64_t n[64];
    if (oracle_levels(N, B, b, L, n, 64) != L) return -1;
    int64_t off[64];
    off[0] = 0;
    for (int l = 1; l < L; ++l) off[l] = off[l - 1] + n[l - 1];
    (void)B;

    int64_t cap = n[0] > n[L - 1] ? n[0] : n[L - 1];
    if (cap < 1) cap = 1;
    if (pr_node) *n_pr = 0;
    scored_t *cand = (scored_t *)malloc(sizeof(scored_t) * (size_t)cap);
    int64_t *kept = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
    int64_t n_keep = 0;

    for (int l = L; l >= 1; --l) {
        int64_t nc = 0;
        if (l == L) {
            for (int64_t i = 0; i < n[L - 1]; ++i) cand[nc++].id = i;
        } else {
            for (int64_t k = 0; k < n_keep; ++k)
                for (int64_t c = kept[k] * b; c < kept[k] * b + b && c < n[l - 1]; ++c)
                    cand[nc++].id = c;
        }
        for (int64_t i = 0; i < nc; ++i) {
            int64_t node = off[l - 1] + cand[i].id;
            double best = -INFINITY;
            int br = 0;
            for (int r = 0; r < R; ++r) {
                double t = scale * dot(q, khat + (node * R + r) * d, d) + bhat[node * R + r];
                if (t > best) { best = t; br = r; }
            }
            cand[i].s = best;
            cand[i].plane = br;
        }
        qsort(cand, (size_t)nc, sizeof(scored_t), cmp_scored);

        int64_t m = nc;
        double mg = INFINITY;
        if (nc > 0 && p[l - 1] < 1.0) {
            double total = 0.0;
            double smax = cand[0].s;
            for (int64_t i = 0; i < nc; ++i) total += exp(cand[i].s - smax);
            double cum = 0.0, prev = 0.0;
            for (m = 0; m < nc;) {
                prev = cum;
                cum += exp(cand[m].s - smax) / total;
                ++m;
                if (cum >= p[l - 1]) break;
            }
            double t1 = cum - p[l - 1];
            double t2 = p[l - 1] - prev;
            double t3 = m < nc ? cand[m - 1].s - cand[m].s : INFINITY;
            mg = t1 < t2 ? t1 : t2;
            if (t3 < mg) mg = t3;
        }
        n_cand[l - 1] = nc;
        n_kept[l - 1] = m;
        margin[l - 1] = mg;
        if (pr_node)
            for (int64_t i = m; i < nc; ++i) {
                pr_node[*n_pr] = off[l - 1] + cand[i].id;
                pr_plane[*n_pr] = cand[i].plane;
                pr_s[*n_pr] = cand[i].s;
                ++*n_pr;
            }
        for (int64_t i = 0; i < m; ++i) kept[i] = cand[i].id;
        qsort(kept, (size_t)m, sizeof(int64_t), cmp_i64);
        n_keep = m;
    }
    for (int64_t i = 0; i < n_keep; ++i) sel[i] = kept[i];
    free(cand);
    free(kept);
    return n_keep;
}

/*
 * The final key set ([HTI] Routing, I(q)): the sink {0} ([EoQ]: the first
 * token is always kept), the keys of the kept level-1 blocks, and the current
 * chunk C_cur(t) = [min(floor(t/B), n_1) * B, t], without duplicates, in
 * ascending order.  idx needs room for t+1 entries.  Returns the count.
 */
int64_t oracle_index_set(const int64_t *sel, int64_t n_sel, int64_t t, int B, int64_t n1,
                         int64_t *idx) {
    char *mark = (char *)calloc((size_t)(t + 1), 1);
    mark[0] = 1;
    for (int64_t k = 0; k < n_sel; ++k)
        for (int64_t j = sel[k] * B; j < sel[k] * B + B && j <= t; ++j) mark[j] = 1;
    int64_t cb = t / B < n1 ? t / B : n1;
    for (int64_t j = cb * B; j <= t; ++j) mark[j] = 1;
    int64_t c = 0;
    for (int64_t j = 0; j <= t; ++j) if (mark[j]) idx[c++] = j;
    free(mark);
    return c;
}

/*
 * Exact softmax attention over the listed keys ([HTI] Routing,
 * o(q) = Attn(q, K_I, V_I)): o = sum_j softmax_j(scale q.k_j) v_j.
 * K, V are one slice [rows][d]; o has d entries.
 */
void oracle_attend(const double *q, const void *K, const void *V, int dtype, int d,
                   const int64_t *idx, int64_t n_idx, double scale, double *o) {
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    if (n_idx <= 0) return;
    double *z = (double *)malloc(sizeof(double) * (size_t)(n_idx > 0 ? n_idx : 1));
    for (int64_t i = 0; i < n_idx; ++i) z[i] = scale * dot_slice(q, K, dtype, idx[i], d);
    double F = lse(z, n_idx);
    for (int64_t i = 0; i < n_idx; ++i) {
        double w = exp(z[i] - F);
        for (int e = 0; e < d; ++e) o[e] += w * elem(V, dtype, idx[i] * d + e);
    }
    free(z);
}

/*
 * Attention with the pruned subtrees' value summaries ([HTI] Future Directions
 * (4)).  Reading: each pruned node n enters the softmax as one pseudo-key with
 * log-mass s_n (its routing score, the tangent estimate of LSE over its keys) and
 * value vhat_n (its plane r*): o = (sum_{i in I} e^{z_i} v_i + sum_n e^{s_n} vhat_n)
 * / (sum_{i in I} e^{z_i} + sum_n e^{s_n}), z_i = scale q.k_i.  Keys of I(q) that
 * also lie under a pruned node (the sink, a current chunk inside the tree) count in
 * both terms, as the index set and the summaries define them.
 * pr_vhat: n_pr rows of d doubles (each pruned node's vhat at its plane).
 */
void oracle_attend_vsum(const double *q, const void *K, const void *V, int dtype, int d,
                        const int64_t *idx, int64_t n_idx, double scale,
                        const double *pr_s, const double *pr_vhat, int64_t n_pr, double *o) {
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    int64_t n = n_idx + n_pr;
    if (n <= 0) return;
    double *z = (double *)malloc(sizeof(double) * (size_t)n);
    for (int64_t i = 0; i < n_idx; ++i) z[i] = scale * dot_slice(q, K, dtype, idx[i], d);
    for (int64_t j = 0; j < n_pr; ++j) z[n_idx + j] = pr_s[j];
    double F = lse(z, n);
    for (int64_t i = 0; i < n_idx; ++i) {
        double w = exp(z[i] - F);
        for (int e = 0; e < d; ++e) o[e] += w * elem(V, dtype, idx[i] * d + e);
    }
    for (int64_t j = 0; j < n_pr; ++j) {
        double w = exp(z[n_idx + j] - F);
        for (int e = 0; e < d; ++e) o[e] += w * pr_vhat[j * d + e];
    }
    free(z);
}
