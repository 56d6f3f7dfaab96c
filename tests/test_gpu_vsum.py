"""Value summaries on the CUDA path against the fp64 oracle, through the C ABI.

"Subquadratic Attention with a Hierarchical Tree-Structured Indexer", Future Directions (4):
pruned subtrees contribute coarse attention outputs.  Reading (the oracle's): every node also
stores vhat, the values pooled with the weights that pool its khat; decoding adds each node the
top-p cut drops as one pseudo-key of log-mass s (its routing score) and value vhat.

Covers the summaries of every level (both dtypes), append against rebuild (bitwise), decoding
against the oracle's attention with the dropped nodes, the closed form (one key per top node:
the output is dense attention), and the refusals (R > 1, chunked prefill, the no-alloc call).
"""
import math

import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O
from tests.zha_parity import MARGIN, SUMMARY_ATOL, TOL_TIGHT_REL, Decoder, assert_status_clean, compare_tree

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    zha.get_status(clear=True)
    yield


def planted(batch, Hq, Hkv, d, N, N_cap, M, n_q, dtype="bf16"):
    dt = W.torch_dtype(dtype)
    K = torch.zeros((batch, Hkv, N_cap, d), dtype=dt)
    V = torch.zeros_like(K)
    Q = torch.zeros((n_q, batch, Hq, d), dtype=dt)
    G = Hq // Hkv
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice("test", s, h, N, d, M, K[s, h], V[s, h], run=min(W.RUN, N // 4))
            Q[:, s, h * G:(h + 1) * G] = W.cluster_queries("test", s, h, G, n_q, cl).to(dt)
    return K, V, Q, W.reference_queries("test", Hkv, 1, d)


def oracle_vtree(K_slice, V_slice, N, cfg, qref_slice):
    return O.build_tree(K_slice, N, cfg.B, cfg.b, qref_slice, scale=cfg.softmax_scale, L_fixed=cfg.L_fixed,
                        V_slice=V_slice)


def compare_vhat(cfg, tree, ot, s, h):
    for l in range(1, ot.L + 1):
        n = ot.n[l - 1]
        off = sum(ot.n[:l - 1])
        g = zha.tree_vhat_view(cfg, tree, l)[s, h, :n].double().cpu().numpy()
        err = np.max(np.abs(g - ot.vhat[off:off + n, 0]))
        assert err <= SUMMARY_ATOL, f"level {l}: vhat err {err:.3g}"


@pytest.mark.parametrize("d,G,dtype,B,b", [(128, 4, "bf16", 64, 16), (64, 2, "f32", 16, 8)])
def test_value_summaries_of_every_level_match_the_oracle(d, G, dtype, B, b):
    batch, Hkv = 2, 2
    N = [60000 + 37, 41234]
    N_cap = 60160
    K, V, Q, qref = planted(batch, G * Hkv, Hkv, d, max(N), N_cap, 24, 1, dtype)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N_cap, dtype=dtype, p=0.95, vsum=1)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), N)
    dec.build()
    torch.cuda.synchronize()
    for s in range(batch):
        for h in range(Hkv):
            ot = oracle_vtree(K[s, h], V[s, h], N[s], cfg, qref[h])
            compare_tree(cfg, dec.tree, ot, s, h)
            compare_vhat(cfg, dec.tree, ot, s, h)
    assert_status_clean()


def test_append_with_value_summaries_matches_rebuild_bitwise():
    d, G, Hkv, batch, B, b = 128, 4, 1, 1, 16, 4
    N0, steps = 16 * 4 * 4 * 3 + 5, 40
    N_cap = N0 + steps + 8
    K, V, _, qref = planted(batch, G * Hkv, Hkv, d, N0 + steps, N_cap, 4, 1)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N_cap, p=0.95, vsum=1)
    Kd, Vd = K.clone(), V.clone()
    Kd[:, :, N0:] = 0
    Vd[:, :, N0:] = 0
    dec = Decoder(cfg, Kd.cuda(), Vd.cuda(), qref.cuda(), [N0])
    dec.build()
    ref = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N0])
    for i in range(steps):
        zha.append(cfg, dec.K, dec.V, K[:, :, N0 + i].contiguous().cuda(), V[:, :, N0 + i].contiguous().cuda(),
                   dec.N, dec.tree)
        ref.N.fill_(N0 + i + 1)
        ref.tree.zero_()
        ref.build()
        torch.cuda.synchronize()
        for l, n in enumerate(O.levels(N0 + i + 1, B, b), start=1):
            va, vb = zha.tree_vhat_view(cfg, dec.tree, l), zha.tree_vhat_view(cfg, ref.tree, l)
            assert torch.equal(va[:, :, :n], vb[:, :, :n]), (i, l)
            ka, ba = zha.tree_level_view(cfg, dec.tree, l)
            kb, bb = zha.tree_level_view(cfg, ref.tree, l)
            assert torch.equal(ka[:, :, :n], kb[:, :, :n]) and torch.equal(ba[:, :, :n], bb[:, :, :n]), (i, l)
    assert_status_clean()


@pytest.mark.parametrize("d,G,dtype,p", [(128, 4, "bf16", 0.9), (128, 2, "bf16", 0.6), (64, 4, "f32", 0.8)])
def test_decode_with_value_summaries_matches_the_oracle(d, G, dtype, p):
    """Queries whose routing is exact beyond the margin (then the dropped nodes are the same):
    the output against the oracle's attention over I(q) plus the dropped nodes."""
    batch, Hkv = 2, 2
    N = [70000 + 37, 51234]
    N_cap = 70144
    K, V, Q, qref = planted(batch, G * Hkv, Hkv, d, max(N), N_cap, 48, 2, dtype)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=N_cap, dtype=dtype, p=p, vsum=1)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), N)
    dec.build()
    trees = {(s, h): oracle_vtree(K[s, h], V[s, h], N[s], cfg, qref[h]) for s in range(batch) for h in range(Hkv)}
    checked = dropped = 0
    for step in range(Q.shape[0]):
        Qs = Q[step].reshape(batch, 1, G * Hkv, d).contiguous()
        dec.route_attend(Qs.cuda())
        sel, cnt, o = dec.results()
        for s in range(batch):
            for hq in range(G * Hkv):
                ot = trees[(s, hq // G)]
                q = Qs[s, 0, hq]
                rt = O.route(q, ot, p)
                g_sel = sel[s, 0, hq, :int(cnt[s, 0, hq])].numpy().astype(np.int64)
                if rt.min_margin <= MARGIN:
                    continue
                assert np.array_equal(g_sel, rt.sel)
                idx = O.index_set(rt.sel, N[s] - 1, cfg.B, ot.n[0])
                ref = O.attend_vsum(q, K[s, hq // G], V[s, hq // G], idx, ot, rt)
                err = float(np.max(np.abs(o[s, 0, hq].numpy() - ref))) / float(np.max(np.abs(ref)))
                assert err <= TOL_TIGHT_REL, f"(s {s}, head {hq}): relative error {err:.3g}"
                checked += 1
                dropped += len(rt.pr_node) > 0
    assert checked >= batch * G * Hkv and dropped >= checked // 2, (checked, dropped)
    assert_status_clean()


def test_value_summaries_are_exact_when_every_top_node_holds_one_key():
    """All keys under each top-level node equal: every node's tangent is exact and its vhat is
    the mean of its values, so the output with the dropped nodes is dense causal attention."""
    d, G, Hkv, B, b = 128, 4, 1, 64, 4
    per_top = B * b * b                      # three-level tree: the top nodes hold 1024 keys
    n_top = 3
    N = n_top * per_top + 5                  # the last 5 keys are the current chunk, past the tree
    gen = torch.Generator().manual_seed(11)
    tops = torch.randn((n_top, d), generator=gen, dtype=torch.float64)
    Kf = torch.cat([tops.repeat_interleave(per_top, 0), torch.randn((5, d), generator=gen, dtype=torch.float64)])
    K = Kf.to(torch.bfloat16).reshape(1, 1, N, d).contiguous()
    V = torch.randn((1, 1, N, d), generator=gen).to(torch.bfloat16)
    qref = W.reference_queries("test", Hkv, 1, d)
    cfg = zha.Config(d=d, Hq=G, Hkv=Hkv, B=B, b=b, batch=1, N_cap=N, p=0.7, vsum=1)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [N])
    dec.build()
    u = tops[0] / tops[0].norm()
    Q = torch.stack([(1.2 + 0.1 * g) * u * math.sqrt(d) + 0.05 * torch.randn(d, generator=gen, dtype=torch.float64)
                     for g in range(G)]).to(torch.bfloat16).reshape(1, 1, G, d).contiguous()
    dec.route_attend(Q.cuda())
    sel, cnt, o = dec.results()
    assert O.levels(N, B, b) == [n_top * b * b, n_top * b, n_top]
    for g in range(G):
        assert int(cnt[0, 0, g]) < N // B and int(sel[0, 0, g, 0]) == 0   # something dropped; the sink's block kept
        dense = O.dense(Q[0, 0, g], K[0, 0], V[0, 0], N - 1)
        err = float(np.max(np.abs(o[0, 0, g].numpy() - dense))) / float(np.max(np.abs(dense)))
        assert err <= TOL_TIGHT_REL, f"head {g}: relative error {err:.3g} against dense attention"
    assert_status_clean()


def test_value_summaries_refusals():
    base = dict(d=128, Hq=8, Hkv=2, B=64, b=16, batch=1, N_cap=8192, vsum=1)
    with pytest.raises(zha.ZhaError):
        zha.tree_bytes(zha.Config(**{**base, "R": 2}))
    with pytest.raises(zha.ZhaError):
        zha.workspace_bytes(zha.Config(**base), 64)   # chunked prefill
    cfg = zha.Config(**base)
    K = torch.zeros((1, 2, 8192, 128), dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros((1, 1, 8, 128), dtype=torch.bfloat16, device="cuda")
    N = torch.full((1,), 100, dtype=torch.int32, device="cuda")
    sel = torch.zeros((1, 1, 8, 128), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, 1, 8), dtype=torch.int32, device="cuda")
    O_ = torch.zeros((1, 1, 8, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(zha.ZhaError):
        zha.attend_noalloc(cfg, K, K, zha.alloc_tree(cfg), Q, N, sel, cnt, O_)
    assert_status_clean()
