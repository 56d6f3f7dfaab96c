"""Chunked prefill through the C ABI (zha_route / zha_attend / zha_dense with
n_q > 1) against the fp64 oracle.

The tree indexes the first N_p keys; query i of the chunk sits at t = N_p + i and
attends to {0} u (its kept blocks) u [n_1 B, t] ("Subquadratic Attention with a
Hierarchical Tree-Structured Indexer", Routing; the causal tail is the current
chunk).  Index sets must be bit-exact wherever the oracle's cut margin exceeds
1e-4; outputs meet the bf16 bar (2e-2 of |o|_inf) against the oracle over the
GPU's own set, and a tight bar of 2^-8 max|v| there: the tensor-core path rounds
the softmax weights to bf16 (relative error <= 2^-9 each, normalised by the sum of
the rounded weights), so the output moves by at most 2^-9 * 2 max|v|.
"""
import dataclasses

import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O
from tests.zha_parity import Report, assert_status_clean, check_queries, oracle_tree

pytestmark = pytest.mark.gpu

TIGHT_OF_V = 2.0 ** -8


def make_case(batch, Hkv, G, d, Np, n_q, p, run=W.RUN, M=None, seq_base=0):
    w = dataclasses.replace(W.WORKLOADS["prefill256k"], batch=batch, Hkv=Hkv, Hq=Hkv * G, d=d, N=Np, p=p,
                            n_clusters=M or max(1, Np // 2048), steps=n_q)
    data = W.planted(w, device="cuda", N_cap=Np + n_q, n_queries=n_q, run=min(run, max(1, Np - 1)),
                     seq_base=seq_base)
    K, V = data["K"], data["V"]
    K[:, :, Np:] = data["k_new"].permute(1, 2, 0, 3)
    V[:, :, Np:] = data["v_new"].permute(1, 2, 0, 3)
    Q = data["Q"].permute(1, 0, 2, 3).contiguous()
    cfg = zha.Config(d=d, Hq=Hkv * G, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=Np + n_q, p=p)
    return w, cfg, K, V, Q, data["qref"]


class Prefill:
    def __init__(self, cfg, K, V, Q, qref, Np, n_q):
        self.cfg, self.K, self.V, self.Q, self.qref = cfg, K, V, Q, qref
        self.Np, self.n_q = Np, n_q
        b = cfg.batch
        self.N = torch.full((b,), Np + n_q, dtype=torch.int32, device="cuda")
        self.tree = zha.alloc_tree(cfg)
        self.ws = zha.alloc_workspace(cfg, n_q)
        self.sel_cap = max(cfg.N_cap // cfg.B, 1)
        self.sel = torch.zeros((b, n_q, cfg.Hq, self.sel_cap), dtype=torch.int32, device="cuda")
        self.cnt = torch.zeros((b, n_q, cfg.Hq), dtype=torch.int32, device="cuda")
        self.O = torch.full((b, n_q, cfg.Hq, cfg.d), float("nan"), dtype=torch.float32, device="cuda")

    def build(self):
        Nb = torch.full((self.cfg.batch,), self.Np, dtype=torch.int32, device="cuda")
        zha.build(self.cfg, self.K, self.qref, Nb, self.tree)

    def run(self):
        zha.route(self.cfg, self.tree, self.Q, self.N, self.sel, self.cnt, self.ws, n_q=self.n_q)
        zha.attend(self.cfg, self.K, self.V, self.tree, self.Q, self.N, self.sel, self.cnt, self.O, self.ws,
                   n_q=self.n_q)

    def dense(self, O):
        zha.dense(self.cfg, self.K, self.V, self.Q, self.N, O, self.ws, n_q=self.n_q)


def check_prefill(pf: Prefill, slices, queries, p, rep=None):
    """Oracle parity of the sampled (sequence, KV head) slices and chunk queries."""
    cfg = pf.cfg
    G = cfg.G
    torch.cuda.synchronize()
    sel, cnt, out = pf.sel.cpu(), pf.cnt.cpu(), pf.O.cpu()
    Qh = pf.Q.cpu()
    rep = rep or Report()
    for (s, h) in slices:
        Kh = pf.K[s, h].cpu()
        Vh = pf.V[s, h].cpu()
        ot = oracle_tree(Kh, pf.Np, cfg, pf.qref[h].cpu())
        for i in queries:
            hs = slice(h * G, (h + 1) * G)
            check_queries(cfg, ot, Kh, Vh, [pf.Np + i] * G, Qh[s, i, hs].float(), sel[s, i, hs], cnt[s, i, hs],
                          out[s, i, hs].numpy(), p, rep, tight_of_v=TIGHT_OF_V)
    return rep


@pytest.mark.parametrize("G,d", [(4, 128), (2, 64), (1, 128)])
def test_prefill_small_matches_oracle(G, d):
    Np, n_q = 40000 + 17, 300            # an incomplete prefix block, a 5-block causal tail
    w, cfg, K, V, Q, qref = make_case(batch=2, Hkv=2, G=G, d=d, Np=Np, n_q=n_q, p=0.95, M=20)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    zha.get_status(clear=True)
    pf.build()
    pf.run()
    rep = check_prefill(pf, [(0, 0), (1, 1)], [0, 1, 63, 64, 150, n_q - 1], 0.95)
    rep.check()
    assert rep.exact_required >= rep.queries // 2, rep
    assert torch.isfinite(pf.O).all()
    assert_status_clean()


def test_prefill_p_one_is_causal_dense_attention():
    """p = 1 keeps every block: the chunk's outputs equal causal dense attention (and
    the in-library dense prefill).  Every row then has ~n_1 blocks, so the plan must
    widen its superblocks to fit the partial slots."""
    Np, n_q = 20000 + 40, 200
    w, cfg, K, V, Q, qref = make_case(batch=1, Hkv=2, G=4, d=128, Np=Np, n_q=n_q, p=1.0, M=8)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    zha.get_status(clear=True)
    pf.build()
    pf.run()
    Od = torch.full_like(pf.O, float("nan"))
    pf.dense(Od)
    torch.cuda.synchronize()
    cnt = pf.cnt.cpu()
    assert (cnt == Np // 64).all()
    o, od = pf.O.cpu().numpy(), Od.cpu().numpy()
    for h in range(cfg.Hkv):
        Kh, Vh = pf.K[0, h].cpu(), pf.V[0, h].cpu()
        vmax = float(Vh[:Np + n_q].float().abs().max())
        for i in (0, 7, 64, 199):
            for g in range(cfg.G):
                hq = h * cfg.G + g
                ref = O.dense(pf.Q[0, i, hq].cpu().float(), Kh, Vh, Np + i)
                assert np.max(np.abs(o[0, i, hq] - ref)) <= TIGHT_OF_V * vmax
                assert np.max(np.abs(od[0, i, hq] - ref)) <= TIGHT_OF_V * vmax
    assert_status_clean()


def test_dense_prefill_matches_oracle_causal_attention():
    Np, n_q = 9000 + 5, 130
    w, cfg, K, V, Q, qref = make_case(batch=2, Hkv=1, G=2, d=64, Np=Np, n_q=n_q, p=0.9, M=4)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    zha.get_status(clear=True)
    pf.dense(pf.O)
    torch.cuda.synchronize()
    o = pf.O.cpu().numpy()
    for s in range(2):
        Kh, Vh = pf.K[s, 0].cpu(), pf.V[s, 0].cpu()
        vmax = float(Vh[:Np + n_q].float().abs().max())
        for i in (0, 1, 65, 129):
            for g in range(2):
                ref = O.dense(pf.Q[s, i, g].cpu().float(), Kh, Vh, Np + i)
                err = np.max(np.abs(o[s, i, g] - ref))
                assert err <= TIGHT_OF_V * vmax, (s, i, g, err)
                assert err <= 2e-2 * np.max(np.abs(ref))
    assert_status_clean()


def test_prefill_without_tree_blocks_is_all_tail():
    """N_p < B: the tree has no complete block, so every query attends causally to [0, t]."""
    Np, n_q = 40, 100
    w, cfg, K, V, Q, qref = make_case(batch=1, Hkv=1, G=4, d=128, Np=Np, n_q=n_q, p=0.9, M=1, run=8)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    zha.get_status(clear=True)
    pf.build()
    pf.run()
    torch.cuda.synchronize()
    assert (pf.cnt.cpu() == 0).all()
    o = pf.O.cpu().numpy()
    Kh, Vh = pf.K[0, 0].cpu(), pf.V[0, 0].cpu()
    vmax = float(Vh[:Np + n_q].float().abs().max())
    for i in (0, 23, 99):
        for g in range(4):
            ref = O.dense(pf.Q[0, i, g].cpu().float(), Kh, Vh, Np + i)
            assert np.max(np.abs(o[0, i, g] - ref)) <= TIGHT_OF_V * vmax
    assert_status_clean()


def test_prefill_refuses_a_tree_that_does_not_end_at_the_chunk():
    Np, n_q = 5000, 64
    w, cfg, K, V, Q, qref = make_case(batch=1, Hkv=1, G=1, d=128, Np=Np, n_q=n_q, p=0.9, M=2)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    Nb = torch.full((1,), Np + 1, dtype=torch.int32, device="cuda")    # one key too many in the tree
    zha.get_status(clear=True)
    zha.build(cfg, K, qref, Nb, pf.tree)
    pf.run()
    bits = zha.get_status(clear=True)
    assert bits & (1 << 1), zha.status_names(bits)


def test_prefill_host_checks():
    cfg = zha.Config(d=128, Hq=8, Hkv=2, B=64, b=16, batch=1, N_cap=4096, p=0.9, dtype="f32")
    with pytest.raises(zha.ZhaError) as e:
        zha.workspace_bytes(cfg, 16)
    assert e.value.code == 2
    cfg = zha.Config(d=128, Hq=8, Hkv=2, B=32, b=16, batch=1, N_cap=4096, p=0.9)
    with pytest.raises(zha.ZhaError) as e:
        zha.workspace_bytes(cfg, 16)
    assert e.value.code == 2


def test_prefill_is_deterministic():
    Np, n_q = 30000, 256
    w, cfg, K, V, Q, qref = make_case(batch=1, Hkv=2, G=4, d=128, Np=Np, n_q=n_q, p=0.95, M=12)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    pf.build()
    pf.run()
    torch.cuda.synchronize()
    first = (pf.sel.clone(), pf.cnt.clone(), pf.O.clone())
    pf.run()
    torch.cuda.synchronize()
    assert torch.equal(first[1], pf.cnt) and torch.equal(first[0], pf.sel)
    assert torch.equal(first[2], pf.O)


def test_causal_chunk_insertion_matches_decode_semantics():
    """The chunk's own blocks inserted causally: the chunk runs in block-aligned sub-chunks and
    zha_extend indexes the blocks completed before each, so query t routes over the tree of the
    keys [0, floor(t/B) B) and attends to its own block up to t -- what decoding it token by token
    would do."""
    Np, n_q, B = 12800, 150, 64            # the prefix ends on a block boundary
    w, cfg, K, V, Q, qref = make_case(batch=1, Hkv=2, G=4, d=128, Np=Np, n_q=n_q, p=0.95, M=8)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    ws_sub = zha.alloc_workspace(cfg, B)
    zha.get_status(clear=True)
    pf.build()
    for i0 in range(0, n_q, B):
        i1 = min(i0 + B, n_q)
        if i0:
            zha.extend(cfg, pf.K, torch.full((1,), Np + i0, dtype=torch.int32, device="cuda"), pf.tree)
        N_end = torch.full((1,), Np + i1, dtype=torch.int32, device="cuda")
        zha.route(cfg, pf.tree, Q[:, i0:i1], N_end, pf.sel[:, i0:i1], pf.cnt[:, i0:i1], ws_sub, n_q=i1 - i0)
        zha.attend(cfg, pf.K, pf.V, pf.tree, Q[:, i0:i1], N_end, pf.sel[:, i0:i1], pf.cnt[:, i0:i1],
                   pf.O[:, i0:i1], ws_sub, n_q=i1 - i0)
    torch.cuda.synchronize()
    sel, cnt, out = pf.sel.cpu(), pf.cnt.cpu(), pf.O.cpu()
    rep = Report()
    for h in range(cfg.Hkv):
        Kh, Vh = pf.K[0, h].cpu(), pf.V[0, h].cpu()
        for i in (0, 63, 64, 100, n_q - 1):
            t = Np + i
            ot = oracle_tree(Kh, (t // B) * B, cfg, pf.qref[h].cpu())
            hs = slice(h * cfg.G, (h + 1) * cfg.G)
            check_queries(cfg, ot, Kh, Vh, [t] * cfg.G, pf.Q[0, i, hs].cpu().float(), sel[0, i, hs], cnt[0, i, hs],
                          out[0, i, hs].numpy(), 0.95, rep, tight_of_v=TIGHT_OF_V)
    rep.check()
    assert rep.exact_required >= rep.queries // 2, rep
    assert_status_clean()


def test_workspace_reused_across_chunk_lengths():
    """One workspace serves chunks of different lengths and then decoding: its layout depends
    on n_q, so what a longer chunk left in it must reach neither a shorter chunk nor a decode
    step (both bit-identical to a fresh workspace)."""
    Np, n_q, short = 9000 + 5, 200, 37
    w, cfg, K, V, Q, qref = make_case(batch=2, Hkv=2, G=2, d=128, Np=Np, n_q=n_q, p=0.95, M=8)
    pf = Prefill(cfg, K, V, Q, qref, Np, n_q)
    zha.get_status(clear=True)
    pf.build()
    pf.run()
    Qs = Q[:, :short].contiguous()
    N_s = torch.full((cfg.batch,), Np + short, dtype=torch.int32, device="cuda")

    def run(ws):
        sel = torch.zeros((cfg.batch, short, cfg.Hq, pf.sel_cap), dtype=torch.int32, device="cuda")
        cnt = torch.zeros((cfg.batch, short, cfg.Hq), dtype=torch.int32, device="cuda")
        out = torch.zeros((cfg.batch, short, cfg.Hq, cfg.d), dtype=torch.float32, device="cuda")
        zha.route(cfg, pf.tree, Qs, N_s, sel, cnt, ws, n_q=short)
        zha.attend(cfg, pf.K, pf.V, pf.tree, Qs, N_s, sel, cnt, out, ws, n_q=short)
        return sel, cnt, out

    reused = run(pf.ws)
    fresh = run(zha.alloc_workspace(cfg, short))
    torch.cuda.synchronize()
    for a, b in zip(reused, fresh):
        assert torch.equal(a, b)

    # then a decode step on the same workspace
    assert pf.ws.numel() >= zha.workspace_bytes(cfg, 1)
    Qd = Q[:, :1].contiguous()
    N_d = torch.full((cfg.batch,), Np + 1, dtype=torch.int32, device="cuda")

    def decode(ws):
        sel = torch.zeros((cfg.batch, 1, cfg.Hq, pf.sel_cap), dtype=torch.int32, device="cuda")
        cnt = torch.zeros((cfg.batch, 1, cfg.Hq), dtype=torch.int32, device="cuda")
        out = torch.zeros((cfg.batch, 1, cfg.Hq, cfg.d), dtype=torch.float32, device="cuda")
        zha.route(cfg, pf.tree, Qd, N_d, sel, cnt, ws)
        zha.attend(cfg, pf.K, pf.V, pf.tree, Qd, N_d, sel, cnt, out, ws)
        return sel, cnt, out

    reused = decode(pf.ws)
    fresh = decode(zha.alloc_workspace(cfg, 1))
    torch.cuda.synchronize()
    for a, b in zip(reused, fresh):
        assert torch.equal(a, b)
    assert_status_clean()
