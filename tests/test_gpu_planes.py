"""Nodes with R > 1 reference queries ("Subquadratic Attention with a
Hierarchical Tree-Structured Indexer", Methodology / Tree Construction: one
tangent per reference query; a node's score is the maximum over its planes;
the pages' models use R = 16) on the CUDA path, against the fp64 oracle: every
plane of every level, routing and attention, append against rebuild, and the
chunked prefill."""
import dataclasses

import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from tests.test_gpu_prefill import Prefill, check_prefill
from tests.zha_parity import Decoder, Report, assert_status_clean, check_queries, compare_tree, oracle_tree

pytestmark = pytest.mark.gpu


def planted(batch, Hkv, G, d, N, N_cap, M, n_q, R, run):
    K = torch.zeros((batch, Hkv, N_cap, d), dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    Q = torch.zeros((n_q, batch, Hkv * G, d), dtype=torch.bfloat16)
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice("test", s, h, N, d, M, K[s, h], V[s, h], run=run)
            Q[:, s, h * G:(h + 1) * G] = W.cluster_queries("test", s, h, G, n_q, cl).to(torch.bfloat16)
    return K, V, Q, W.reference_queries("test", Hkv, R, d)


@pytest.mark.parametrize("R", [2, 16])
def test_planes_route_attend(R):
    batch, Hkv, G, d, N = 1, 2, 4, 128, 60013
    K, V, Q, qref = planted(batch, Hkv, G, d, N, N + 64, 24, 2, R, run=4096)
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=N + 64, p=0.95, R=R)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N])
    dec.build()
    trees = {h: oracle_tree(K[0, h], N, cfg, qref[h]) for h in range(Hkv)}
    torch.cuda.synchronize()
    for h, ot in trees.items():
        assert ot.R == R
        compare_tree(cfg, dec.tree, ot, 0, h)
    rep = Report()
    for step in range(Q.shape[0]):
        Qs = Q[step].reshape(batch, 1, Hkv * G, d).contiguous()
        dec.route_attend(Qs.cuda())
        sel, cnt, o = dec.results()
        for hq in range(Hkv * G):
            h = hq // G
            check_queries(cfg, trees[h], K[0, h], V[0, h], N - 1, Qs[0, 0, hq:hq + 1], [sel[0, 0, hq].numpy()],
                          [int(cnt[0, 0, hq])], [o[0, 0, hq].numpy()], 0.95, rep)
    rep.check()
    assert rep.exact_required >= rep.queries // 2, rep
    assert_status_clean()


def test_planes_append_matches_rebuild():
    """R = 3: appended trees equal rebuilt ones bit for bit on every plane."""
    batch, Hkv, G, d, B, b, R = 1, 2, 2, 64, 16, 4, 3
    N0, steps = 1000, 40
    N_cap = N0 + steps + 8
    K, V, Q, qref = planted(batch, Hkv, G, d, N0 + steps, N_cap, 3, 1, R, run=200)
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N_cap, p=0.9, R=R)
    Kd, Vd = K.clone(), V.clone()
    Kd[:, :, N0:] = 0
    Vd[:, :, N0:] = 0
    dec = Decoder(cfg, Kd.cuda(), Vd.cuda(), qref.cuda(), [N0])
    dec.build()
    ref = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N0])
    from oracle import oracle as O
    for i in range(steps):
        zha.append(cfg, dec.K, dec.V, K[:, :, N0 + i].contiguous().cuda(), V[:, :, N0 + i].contiguous().cuda(),
                   dec.N, dec.tree)
        n_now = N0 + i + 1
        ref.N.fill_(n_now)
        ref.tree.zero_()
        ref.build()
        torch.cuda.synchronize()
        lv = O.levels(n_now, B, b)
        for l in range(1, len(lv) + 1):
            ka, ba = zha.tree_level_view(cfg, dec.tree, l)
            kb, bb = zha.tree_level_view(cfg, ref.tree, l)
            n = lv[l - 1]
            assert torch.equal(ka[:, :, :n], kb[:, :, :n]), (i, l)
            assert torch.equal(ba[:, :, :n], bb[:, :, :n]), (i, l)
    assert_status_clean()


def test_planes_prefill():
    R, batch, Hkv, G, d, Np, n_q = 4, 1, 2, 4, 128, 30000 + 9, 200
    w = dataclasses.replace(W.WORKLOADS["prefill256k"], batch=batch, Hkv=Hkv, Hq=Hkv * G, d=d, N=Np, p=0.95,
                            n_clusters=12, steps=n_q, R=R)
    data = W.planted(w, device="cuda", N_cap=Np + n_q, n_queries=n_q, run=4096)
    K, V = data["K"], data["V"]
    K[:, :, Np:] = data["k_new"].permute(1, 2, 0, 3)
    V[:, :, Np:] = data["v_new"].permute(1, 2, 0, 3)
    Q = data["Q"].permute(1, 0, 2, 3).contiguous()
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=Np + n_q, p=0.95, R=R)
    pf = Prefill(cfg, K, V, Q, data["qref"], Np, n_q)
    zha.get_status(clear=True)
    pf.build()
    pf.run()
    rep = check_prefill(pf, [(0, 0), (0, 1)], [0, 1, 100, n_q - 1], 0.95)
    rep.check()
    assert rep.exact_required >= rep.queries // 2, rep
    assert_status_clean()
