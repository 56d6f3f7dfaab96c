"""The pages' tree geometries and per-level top-p schedules on the CUDA path,
against the fp64 oracle.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer":
Methodology / Tree Construction names C-ary trees with one C as chunk size and
fan-out and a fixed depth (C4-L6: 4^6 = 4096 keys per top node; C256-L1: one
level of 256-key chunks); its latency predictions use C8 with p = 0.75; Future
Directions (5) asks for top-p scaled per level with depth (p^{1/L} and others).
Each case builds the tree (every level compared), routes decode queries (index
sets bit-exact beyond the margin) and attends (output bars), and for C4-L6
appends tokens one by one against rebuilds.
"""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O
from tests.zha_parity import Decoder, Report, assert_status_clean, check_queries, compare_tree, oracle_tree

pytestmark = pytest.mark.gpu

GEOMETRIES = {
    # name: (B, b, L_fixed, p, N, clusters)
    "C4-L6": (4, 4, 6, 0.95, 4 ** 6 * 6 + 13, 8),
    "C8-p0.75": (8, 8, 0, 0.75, 30011, 12),
    "C256-L1": (256, 16, 1, 0.95, 100077, 40),
    "p^(1/L)": (64, 16, 0, [0.95 ** (1.0 / 3.0)] * 3, 200005, 96),
    "p-rising-with-depth": (64, 16, 0, [0.9, 0.97, 0.99], 200005, 96),
}


def planted(name, batch, Hkv, G, d, N, N_cap, M, n_q, run):
    K = torch.zeros((batch, Hkv, N_cap, d), dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    Q = torch.zeros((n_q, batch, Hkv * G, d), dtype=torch.bfloat16)
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice(name, s, h, N, d, M, K[s, h], V[s, h], run=run)
            Q[:, s, h * G:(h + 1) * G] = W.cluster_queries(name, s, h, G, n_q, cl).to(torch.bfloat16)
    return K, V, Q, W.reference_queries(name, Hkv, 1, d)


@pytest.mark.parametrize("name", sorted(GEOMETRIES))
def test_geometry_route_attend(name):
    B, b, L_fixed, p, N, M = GEOMETRIES[name]
    batch, Hkv, G, d = 1, 2, 4, 128
    K, V, Q, qref = planted("test", batch, Hkv, G, d, N, N + 64, M, 2, run=min(W.RUN, N // 8))
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N + 64, p=p, L_fixed=L_fixed)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N])
    dec.build()
    trees = {h: oracle_tree(K[0, h], N, cfg, qref[h]) for h in range(Hkv)}
    torch.cuda.synchronize()
    for h, ot in trees.items():
        if L_fixed:
            assert ot.L == L_fixed
        compare_tree(cfg, dec.tree, ot, 0, h)
    rep = Report()
    for step in range(Q.shape[0]):
        Qs = Q[step].reshape(batch, 1, Hkv * G, d).contiguous()
        dec.route_attend(Qs.cuda())
        sel, cnt, o = dec.results()
        for hq in range(Hkv * G):
            h = hq // G
            check_queries(cfg, trees[h], K[0, h], V[0, h], N - 1, Qs[0, 0, hq:hq + 1], [sel[0, 0, hq].numpy()],
                          [int(cnt[0, 0, hq])], [o[0, 0, hq].numpy()], p, rep)
    rep.check()
    assert rep.exact_required >= rep.queries // 2, rep
    assert_status_clean()


def test_c4_l6_append_matches_rebuild():
    """C4-L6 with appends: a leaf completes every 4 tokens and its six-level ancestor path is
    recomputed; the tree equals a fresh build at every step, bit for bit."""
    B, b, L_fixed = 4, 4, 6
    batch, Hkv, G, d = 1, 1, 2, 128
    N0, steps = 4096 * 2 + 3, 21
    N_cap = N0 + steps + 8
    K, V, Q, qref = planted("test", batch, Hkv, G, d, N0 + steps, N_cap, 4, 1, run=512)
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N_cap, p=0.95, L_fixed=L_fixed)
    Kd, Vd = K.clone(), V.clone()
    Kd[:, :, N0:] = 0
    Vd[:, :, N0:] = 0
    dec = Decoder(cfg, Kd.cuda(), Vd.cuda(), qref.cuda(), [N0])
    dec.build()
    ref = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N0])
    for i in range(steps):
        zha.append(cfg, dec.K, dec.V, K[:, :, N0 + i].contiguous().cuda(), V[:, :, N0 + i].contiguous().cuda(),
                   dec.N, dec.tree)
        n_now = N0 + i + 1
        ref.N.fill_(n_now)
        ref.tree.zero_()
        ref.build()
        torch.cuda.synchronize()
        lv = O.levels(n_now, B, b, L_fixed)
        assert len(lv) == L_fixed
        for l in range(1, L_fixed + 1):
            ka, ba = zha.tree_level_view(cfg, dec.tree, l)
            kb, bb = zha.tree_level_view(cfg, ref.tree, l)
            n = lv[l - 1]
            assert torch.equal(ka[:, :, :n], kb[:, :, :n]), (i, l)
            assert torch.equal(ba[:, :, :n], bb[:, :, :n]), (i, l)
    assert_status_clean()
