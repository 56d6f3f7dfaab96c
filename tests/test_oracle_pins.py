"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Pages: [HTI] "Subquadratic Attention with a Hierarchical Tree-Structured
Indexer"; [EoQ] "Zyphra Hierarchical Attention: The End of Quadratic
Attention?".  None of these tests trusts the oracle's own formulas: each one
checks a closed form, a limit that reduces to a textbook computation done here
with numpy/scipy, a brute-force enumeration, or values written out by hand.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


def softmax(z):
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


# ---------------------------------------------------------------- geometry

def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


def test_geometry_golden():
    """Nodes per level match the pages' worked geometries and the workload depths."""
    cases = 0
    for line in _golden_lines("geometry.txt"):
        lhs, rest = line.split(":")
        N, B, b, Lf = (int(x) for x in lhs.split())
        expect = [int(x) for x in rest.split("|")[0].split()]
        assert O.levels(N, B, b, Lf) == expect, line
        cases += 1
    assert cases >= 7


def test_geometry_span_c4_l6():
    """C4-L6: a top node spans C^L = 4096 keys ([HTI] Robustness to Geometry)."""
    n = O.levels(4096 * 3, 4, 4, 6)
    assert n[-1] == 3 and 4 * 4 ** 5 == 4096


# ---------------------------------------------------------------- leaf summaries

def _tree(K, N, B, b, R=1, L_fixed=0, seed=1):
    d = K.shape[1]
    q = rng(seed).standard_normal((16, R, d)) / math.sqrt(d)
    return O.build_tree(K.astype(np.float32), N, B, b, q, L_fixed=L_fixed), q


def test_leaf_tangent_touches_lse_at_reference_query():
    """t_r(qhat_r) = F_C(qhat_r) exactly ([HTI] Tree Construction: first-order Taylor at qhat_r)."""
    d, B, b, N = 32, 16, 4, 16 * 20
    K = rng(2).standard_normal((N, d)).astype(np.float32).astype(np.float64)
    tree, q = _tree(K, N, B, b)
    kh, bh = tree.level(1)
    sc = 1 / math.sqrt(d)
    for j in range(tree.n[0]):
        F = logsumexp(sc * K[j * B:(j + 1) * B] @ q[0, 0])
        t = sc * q[0, 0] @ kh[j, 0] + bh[j, 0]
        assert abs(t - F) < 1e-12


def test_leaf_tangent_gradient_matches_lse_gradient():
    """grad F_C(qhat) = khat / sqrt(d): pins the softmax-weighted pooling of the keys."""
    d, B, b, N = 16, 8, 4, 8 * 5
    K = rng(3).standard_normal((N, d)).astype(np.float32).astype(np.float64)
    tree, q = _tree(K, N, B, b)
    kh, _ = tree.level(1)
    sc = 1 / math.sqrt(d)
    eps = 1e-5
    for j in range(tree.n[0]):
        Kj = K[j * B:(j + 1) * B]
        g = np.array([(logsumexp(sc * Kj @ (q[0, 0] + eps * e)) - logsumexp(sc * Kj @ (q[0, 0] - eps * e)))
                      / (2 * eps) for e in np.eye(d)])
        assert np.max(np.abs(g - kh[j, 0] * sc)) < 1e-8


def test_leaf_tangent_is_lower_bound():
    """LSE is convex, so every tangent lies below F_C at any query."""
    d, B, b, N = 32, 16, 4, 16 * 8
    K = rng(4).standard_normal((N, d))
    tree, _ = _tree(K, N, B, b)
    kh, bh = tree.level(1)
    sc = 1 / math.sqrt(d)
    for x in rng(5).standard_normal((50, d)) * 2:
        for j in range(tree.n[0]):
            F = logsumexp(sc * K[j * B:(j + 1) * B].astype(np.float32).astype(np.float64) @ x)
            assert sc * x @ kh[j, 0] + bh[j, 0] <= F + 1e-12


def test_leaf_block_of_one_key_is_the_key():
    """With B = 1: khat = k and bhat = 0, so the score is q.k/sqrt(d) exactly."""
    d, N = 8, 12
    K = rng(6).standard_normal((N, d)).astype(np.float32)
    tree, _ = _tree(K, N, 1, 16)
    kh, bh = tree.level(1)
    assert np.array_equal(kh[:, 0], K.astype(np.float64))
    assert np.max(np.abs(bh)) < 1e-15


def test_bf16_keys_are_widened_exactly():
    """bf16 storage: the oracle reads bf16 bits as the same values as their fp32 widening."""
    import torch
    d, B, b, N = 16, 8, 4, 8 * 6
    Kb = torch.randn((N, d), generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    q = rng(7).standard_normal((16, 1, d)) / 4
    t1 = O.build_tree(Kb, N, B, b, q)
    t2 = O.build_tree(Kb.float(), N, B, b, q)
    assert np.array_equal(t1.khat, t2.khat) and np.array_equal(t1.bhat, t2.bhat)


# ---------------------------------------------------------------- upper levels

def _children_scores(tree, l, x):
    """Log-mass estimates s_c(x) = max_r tangent of the level-(l-1) nodes, a [n_{l-1}] vector."""
    kh, bh = tree.level(l - 1)
    sc = tree.scale
    return np.max(sc * np.einsum("nrd,d->nr", kh, x) + bh, axis=1)


@pytest.mark.parametrize("R", [1, 2])
def test_upper_tangent_touches_children_lse(R):
    """A level-l plane r is the tangent of LSE_c s_c at qhat_{l,r}: equal there, gradient k-hat/sqrt(d)."""
    d, B, b, N = 16, 4, 4, 4 * 4 * 4 * 3 + 8
    K = rng(8).standard_normal((N, d))
    tree, q = _tree(K, N, B, b, R=R)
    assert tree.n == [50, 13, 4]       # partial last parents at levels 2 and 3
    eps = 1e-5
    for l in range(2, tree.L + 1):
        kh, bh = tree.level(l)
        nc = tree.n[l - 2]
        for i in range(tree.n[l - 1]):
            c0, c1 = i * b, min(i * b + b, nc)
            for r in range(R):
                x = q[l - 1, r]
                F = logsumexp(_children_scores(tree, l, x)[c0:c1])
                t = tree.scale * x @ kh[i, r] + bh[i, r]
                assert abs(t - F) < 1e-12
                g = np.array([(logsumexp(_children_scores(tree, l, x + eps * e)[c0:c1])
                               - logsumexp(_children_scores(tree, l, x - eps * e)[c0:c1])) / (2 * eps)
                              for e in np.eye(d)])
                assert np.max(np.abs(g - kh[i, r] * tree.scale)) < 1e-7


def test_upper_level_over_single_keys_is_a_leaf_summary():
    """With B = 1 the level-2 node over b single keys equals the level-1 summary of a B=b tree."""
    d, b, N = 16, 4, 4 * 9
    K = rng(9).standard_normal((N, d)).astype(np.float32)
    q = rng(10).standard_normal((16, 1, d)) / 4
    t1 = O.build_tree(K, N, 1, b, q, L_fixed=2)           # level 2 = groups of b keys
    q2 = q.copy()
    q2[0] = q[1]                                          # the B=b tree's leaf uses the same query
    t2 = O.build_tree(K, N, b, b, q2, L_fixed=1)
    kh1, bh1 = t1.level(2)
    kh2, bh2 = t2.level(1)
    assert np.max(np.abs(kh1 - kh2)) < 1e-12 and np.max(np.abs(bh1 - bh2)) < 1e-12


def test_every_level_is_a_lower_bound_of_the_raw_keys_lse():
    """Each node's estimate s(x) <= LSE of the raw keys it spans, at every level."""
    d, B, b, N = 16, 4, 3, 4 * 3 * 3 * 3 + 5
    K = rng(11).standard_normal((N, d))
    tree, _ = _tree(K, N, B, b, R=2)
    Kf = K.astype(np.float32).astype(np.float64)
    for x in rng(12).standard_normal((20, d)) * 2:
        for l in range(1, tree.L + 1):
            kh, bh = tree.level(l)
            span = B * b ** (l - 1)
            for i in range(tree.n[l - 1]):
                lo, hi = i * span, min((i + 1) * span, tree.n[0] * B)
                F = logsumexp(tree.scale * Kf[lo:hi] @ x)
                s = np.max(tree.scale * kh[i] @ x + bh[i])
                assert s <= F + 1e-10


# ---------------------------------------------------------------- routing

def brute_top_p(probs, p):
    """Smallest set of indices whose probabilities reach p, largest first, ties to the lower index."""
    order = sorted(range(len(probs)), key=lambda i: (-probs[i], i))
    acc, out = 0.0, []
    for i in order:
        out.append(i)
        acc += probs[i]
        if acc >= p:
            break
    return sorted(out)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("p", [0.5, 0.8, 0.95])
def test_flat_routing_is_the_top_p_set_of_attention(seed, p):
    """B = 1, one level: routing keeps the top-p set of the full attention probabilities ([HTI] Key Insight)."""
    d, N = 16, 12
    r = rng(100 + seed)
    K = (r.standard_normal((N, d)) * 1.5).astype(np.float32)
    x = r.standard_normal(d) * 2
    tree, _ = _tree(K, N, 1, 16)
    assert tree.L == 1
    probs = softmax(tree.scale * K.astype(np.float64) @ x)
    assert list(O.route(x, tree, p).sel) == brute_top_p(list(probs), p)


@pytest.mark.parametrize("seed", range(4))
def test_open_upper_levels_reduce_to_flat_top_p(seed):
    """B = 1, several levels, p = 1 above level 1: level 1 sees every key, so it is flat top-p."""
    d, N, b = 16, 40, 3
    r = rng(200 + seed)
    K = (r.standard_normal((N, d)) * 1.5).astype(np.float32)
    x = r.standard_normal(d) * 2
    tree, _ = _tree(K, N, 1, b)
    assert tree.L >= 3
    p = [0.9] + [1.0] * (tree.L - 1)
    probs = softmax(tree.scale * K.astype(np.float64) @ x)
    rt = O.route(x, tree, p)
    assert list(rt.sel) == brute_top_p(list(probs), 0.9)
    assert list(rt.n_cand) == [N] + tree.n[1:]


def test_ties_go_to_the_lower_id():
    """Equal scores are ordered by node id, so the cut keeps the lower ids."""
    d, N = 8, 10
    K = np.zeros((N, d), dtype=np.float32)
    K[:, 0] = 1.0                      # all ten keys identical: equal scores
    x = np.zeros(d)
    x[0] = 1.0
    tree, _ = _tree(K, N, 1, 16)
    for p, keep in [(0.1, 1), (0.35, 4), (0.7, 7), (1.0, 10)]:
        assert list(O.route(x, tree, p).sel) == list(range(keep))
    K[7, 0] = 2.0                      # one strictly larger key goes first
    tree, _ = _tree(K, N, 1, 16)
    sel = list(O.route(x, tree, 0.5).sel)
    assert 7 in sel and sel[0] == 0 and len(sel) < N


def test_upper_level_cut_expands_only_kept_children():
    """Two levels, p < 1 at the top and 1 below: the kept leaves are exactly the children of the
    brute-force top-p set of the top level's estimates (partial last parent included)."""
    d, b = 16, 4
    N = 4 * 6 + 2                      # 26 single-key leaves, 7 parents, the last with 2 children
    for seed in range(5):
        r = rng(300 + seed)
        K = (r.standard_normal((N, d)) * 1.5).astype(np.float32)
        x = r.standard_normal(d) * 2
        tree, _ = _tree(K, N, 1, b, L_fixed=2)
        s_top = _children_scores_level(tree, 2, x)
        kept_top = brute_top_p(list(softmax(s_top)), 0.8)
        expect = [c for i in kept_top for c in range(i * b, min(i * b + b, N))]
        rt = O.route(x, tree, [1.0, 0.8])
        assert list(rt.sel) == expect


def _children_scores_level(tree, l, x):
    kh, bh = tree.level(l)
    return np.max(tree.scale * np.einsum("nrd,d->nr", kh, x) + bh, axis=1)


def test_margin_is_the_distance_of_the_cut_from_p():
    """For a flat one-level case the margin equals min(c_m - p, p - c_{m-1}, s_(m) - s_(m+1))
    computed here from brute-force sorted probabilities and scores."""
    d, N = 16, 12
    r = rng(400)
    K = (r.standard_normal((N, d)) * 1.5).astype(np.float32)
    x = r.standard_normal(d) * 2
    tree, _ = _tree(K, N, 1, 16)
    z = np.sort(tree.scale * K.astype(np.float64) @ x)[::-1]
    probs = softmax(z)
    c = np.cumsum(probs)
    m = int(np.argmax(c >= 0.8)) + 1
    expect = min(c[m - 1] - 0.8, 0.8 - (c[m - 2] if m >= 2 else 0.0), z[m - 1] - z[m])
    assert abs(O.route(x, tree, 0.8).margin[0] - expect) < 1e-12


# ---------------------------------------------------------------- index set and attention

def _ranges(text):
    out = []
    for tok in text.split():
        if "-" in tok:
            a, b_ = tok.split("-")
            out.extend(range(int(a), int(b_) + 1))
        else:
            out.append(int(tok))
    return out


def test_index_set_golden():
    n = 0
    for line in _golden_lines("index_sets.txt"):
        lhs, rhs = line.split(":")
        B, n1, t, sel = lhs.split()
        sel = [] if sel == "-" else [int(s) for s in sel.split(",")]
        got = O.index_set(sel, int(t), int(B), int(n1))
        assert list(got) == _ranges(rhs), line
        n += 1
    assert n >= 9


def test_attention_matches_numpy_softmax():
    d, N = 32, 50
    r = rng(500)
    K = r.standard_normal((N, d)).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    x = r.standard_normal(d)
    idx = np.array([0, 3, 4, 17, 49])
    sc = 1 / math.sqrt(d)
    w = softmax(sc * K[idx].astype(np.float64) @ x)
    expect = w @ V[idx].astype(np.float64)
    assert np.max(np.abs(O.attend(x, K, V, idx) - expect)) < 1e-13


def test_p_one_routes_every_key_and_equals_dense_attention():
    """p = 1 keeps every candidate at every level, so I(q) = [0, t] and o = dense attention."""
    d, B, b, N = 16, 4, 3, 4 * 3 * 3 * 2 + 3
    r = rng(600)
    K = r.standard_normal((N, d)).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    tree, _ = _tree(K, N, B, b)
    x = r.standard_normal(d) * 3
    t = N - 1
    rt, idx, o = O.decode_query(x, tree, K, V, t, 1.0)
    assert list(rt.sel) == list(range(tree.n[0]))
    assert list(idx) == list(range(N))
    w = softmax(tree.scale * K.astype(np.float64) @ x)
    assert np.max(np.abs(o - w @ V.astype(np.float64))) < 1e-13


def test_prefill_query_with_p_one_is_causal_dense_attention():
    """Chunked prefill reading: a tree over the first N_p keys only, a chunk query at
    t > N_p.  With p = 1 every tree block is kept and the causal tail [n_1 B, t]
    completes the set, so I(q) = [0, t] and o is causal dense attention up to t."""
    d, B, b, Np, n_chunk = 16, 4, 3, 4 * 3 * 3 * 2 + 2, 9
    r = rng(610)
    K = r.standard_normal((Np + n_chunk, d)).astype(np.float32)
    V = r.standard_normal((Np + n_chunk, d)).astype(np.float32)
    tree, _ = _tree(K, Np, B, b)
    assert tree.n[0] * B < Np          # an incomplete prefix block stays out of the tree
    for i in (0, 4, n_chunk - 1):
        t = Np + i
        x = r.standard_normal(d) * 3
        rt, idx, o = O.decode_query(x, tree, K, V, t, 1.0)
        assert list(idx) == list(range(t + 1))
        w = softmax(tree.scale * K[:t + 1].astype(np.float64) @ x)
        assert np.max(np.abs(o - w @ V[:t + 1].astype(np.float64))) < 1e-13


@pytest.mark.parametrize("which", ["flat_top_p", "routed"])
def test_eq1_decomposition_holds_with_the_actual_mass(which):
    """[HTI] Key Insight, eq. 1: Attn(q,K,V) = p*.Attn(q,K_S,V_S) + (1-p*).Attn(q,K_Sbar,V_Sbar),
    exact when p* is the attention mass that S actually holds."""
    d, B, b, N = 16, 4, 4, 200
    r = rng(700)
    K = (r.standard_normal((N, d)) * 1.3).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    x = r.standard_normal(d) * 3
    t = N - 1
    sc = 1 / math.sqrt(d)
    probs = softmax(sc * K[:t + 1].astype(np.float64) @ x)
    if which == "flat_top_p":
        S = np.array(brute_top_p(list(probs), 0.9))
    else:
        tree, _ = _tree(K, N, B, b)
        _, S, _ = O.decode_query(x, tree, K, V, t, 0.9)
    Sbar = np.setdiff1d(np.arange(t + 1), S)
    pstar = probs[S].sum()
    full = O.attend(x, K, V, np.arange(t + 1))
    split = pstar * O.attend(x, K, V, S) + (1 - pstar) * O.attend(x, K, V, Sbar)
    assert np.max(np.abs(full - split)) < 1e-12


# ---------------------------------------------------------------- value summaries
# [HTI] Future Directions (4): pruned subtrees contribute coarse attention outputs.
# Reading: vhat pools the values with the weights that pool khat; a pruned node enters the
# softmax as one pseudo-key of log-mass s (its routing score) and value vhat.

def test_value_summary_of_a_uniform_block_is_its_mean_value():
    """A leaf whose keys are all equal gives every key the same weight: vhat is the plain
    mean of the block's values; a block of one key summarises to that key's value."""
    d, B, b = 8, 4, 4
    r = rng(900)
    k = r.standard_normal(d).astype(np.float32)
    K = np.tile(k, (B * 2, 1))
    V = r.standard_normal((B * 2, d)).astype(np.float32)
    tree = O.build_tree(K, B * 2, B, b, r.standard_normal((4, 1, d)), V_slice=V)
    for j in range(2):
        assert np.max(np.abs(tree.vhat[j, 0] - V[j * B:(j + 1) * B].astype(np.float64).mean(0))) < 1e-14
    K1 = r.standard_normal((5, d)).astype(np.float32)
    V1 = r.standard_normal((5, d)).astype(np.float32)
    t1 = O.build_tree(K1, 5, 1, 2, r.standard_normal((8, 1, d)), V_slice=V1)
    assert np.max(np.abs(t1.vhat[:5, 0] - V1.astype(np.float64))) == 0.0


@pytest.mark.parametrize("seed,p", [(0, 0.5), (1, 0.8), (2, 0.95), (3, 0.3)])
def test_kept_blocks_and_pruned_subtrees_partition_the_tree(seed, p):
    d, B, b, N = 8, 4, 4, 4 * 4 * 4 * 5 + 2
    r = rng(910 + seed)
    K = (r.standard_normal((N, d)) * 2).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    tree = O.build_tree(K, N, B, b, r.standard_normal((4, 1, d)), V_slice=V)
    rt = O.route(r.standard_normal(d) * 2, tree, p)
    offs = np.cumsum([0] + tree.n)
    cover = np.zeros(tree.n[0], dtype=int)
    cover[rt.sel] += 1
    for node in rt.pr_node:
        lvl = int(np.searchsorted(offs, node, side="right"))   # 1-based level
        i = int(node - offs[lvl - 1])
        span = b ** (lvl - 1)
        cover[i * span:min((i + 1) * span, tree.n[0])] += 1
    assert (cover == 1).all()


@pytest.mark.parametrize("p", [0.3, 0.6, 0.9])
def test_summaries_are_exact_when_every_top_node_holds_one_key(p):
    """Keys equal under each top-level node make every tangent exact (a node's log-mass is
    scale q.k + log(count), its vhat the mean of its values): attention over I(q) plus the
    pruned nodes then equals dense causal attention for any p, while I(q) alone does not.
    The query favours the sink's node, so key 0 is never also counted inside a pruned node."""
    d, B, b = 8, 4, 4
    r = rng(920)
    n_top, per_top = 3, B * b * b           # three level-3 nodes of 64 keys
    N = n_top * per_top + 3                 # C_cur = the last 3 keys, past the tree
    tops = r.standard_normal((n_top, d))
    K = np.concatenate([np.repeat(tops, per_top, axis=0), r.standard_normal((3, d))]).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    tree = O.build_tree(K, N, B, b, r.standard_normal((4, 1, d)), V_slice=V)
    assert tree.L == 3
    q = 0.6 * tops[0] / np.linalg.norm(tops[0]) * math.sqrt(d) + 0.1 * r.standard_normal(d)
    rt, idx, o = O.decode_query_vsum(q, tree, K, V, N - 1, p)
    assert 0 in rt.sel and len(rt.pr_node) > 0
    dense = O.attend(q, K, V, np.arange(N))
    assert np.max(np.abs(o - dense)) < 1e-12
    assert np.max(np.abs(O.attend(q, K, V, idx) - dense)) > 1e-4


def test_summaries_vanish_at_p_one():
    d, B, b, N = 8, 4, 4, 150
    r = rng(930)
    K = r.standard_normal((N, d)).astype(np.float32)
    V = r.standard_normal((N, d)).astype(np.float32)
    tree = O.build_tree(K, N, B, b, r.standard_normal((4, 1, d)), V_slice=V)
    q = r.standard_normal(d)
    rt, idx, o = O.decode_query_vsum(q, tree, K, V, N - 1, 1.0)
    assert len(rt.pr_node) == 0
    assert np.max(np.abs(o - O.attend(q, K, V, idx))) == 0.0


@pytest.mark.parametrize("R", [1, 2])
def test_value_summaries_pool_with_the_key_summaries_weights(R):
    """With values a linear map of the keys (V = K M), pooling V with khat's weights (and the
    children's best planes) gives vhat = khat M at every level and plane; any other weights
    (uniform, another plane) break it."""
    d, B, b, N = 8, 4, 4, 4 * 4 * 4 * 3 + 6
    r = rng(940 + R)
    K = (r.standard_normal((N, d)) * 1.5).astype(np.float64)
    M = r.standard_normal((d, d))
    tree = O.build_tree(K.astype(np.float32), N, B, b, r.standard_normal((4, R, d)),
                        V_slice=(K.astype(np.float32).astype(np.float64) @ M).astype(np.float32))
    # the oracle widens V from fp32: compare against khat of the same fp32 keys, mapped by M,
    # to the rounding of V to fp32
    Vf = (K.astype(np.float32).astype(np.float64) @ M).astype(np.float32).astype(np.float64)
    err_v = np.abs(Vf - K.astype(np.float32).astype(np.float64) @ M).max()
    assert np.max(np.abs(tree.vhat - tree.khat @ M)) < 4 * err_v + 1e-12
