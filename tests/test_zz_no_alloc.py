"""zha_attend_noalloc, the decode attention entry point for callers that cannot
allocate device memory (a host framework that owns every device allocation and
offers the library none, or a serving path that must not call cudaMalloc): it
runs on the library's static device scratch instead of a caller's workspace.

Collected last on purpose: the static scratch keeps whatever the previous call
left, so this file also checks that results do not depend on what ran before.
It must pass alone in a fresh process and after every other test.
"""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from tests.zha_parity import Report, check_queries, oracle_tree

pytestmark = pytest.mark.gpu


def _case(batch, Hkv, G, d, N, seed_base):
    dt = torch.bfloat16
    K = torch.zeros((batch, Hkv, N, d), dtype=dt)
    V = torch.zeros_like(K)
    Q = torch.zeros((batch, 1, G * Hkv, d), dtype=dt)
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice("test", seed_base + s, h, N, d, 16, K[s, h], V[s, h], run=N // 8)
            Q[s, 0, h * G:(h + 1) * G] = W.cluster_queries("test", seed_base + s, h, G, 1, cl)[0].to(dt)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=N, p=0.95)
    Nt = torch.full((batch,), N, dtype=torch.int32, device="cuda")
    tree = zha.alloc_tree(cfg)
    ws = zha.alloc_workspace(cfg)
    sel = torch.zeros((batch, 1, G * Hkv, N // 64), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((batch, 1, G * Hkv), dtype=torch.int32, device="cuda")
    qref = W.reference_queries("test", Hkv, 1, d)
    zha.build(cfg, K.cuda(), qref.cuda(), Nt, tree)
    return dict(cfg=cfg, K=K, V=V, Q=Q, Kd=K.cuda(), Vd=V.cuda(), Qd=Q.cuda(), N=Nt, tree=tree, ws=ws, sel=sel,
                cnt=cnt, qref=qref)


def _noalloc(c):
    O = torch.full((c["cfg"].batch, 1, c["cfg"].Hq, c["cfg"].d), float("nan"), dtype=torch.float32, device="cuda")
    zha.attend_noalloc(c["cfg"], c["Kd"], c["Vd"], c["tree"], c["Qd"], c["N"], c["sel"], c["cnt"], O)
    torch.cuda.synchronize()
    return O.cpu()


def test_attend_noalloc_matches_attend_twice_in_a_row():
    """Bit for bit the output of zha_attend (the same plan and kernels run on the static scratch
    instead of a workspace), on two calls in a row, after a call of another shape has left its
    items, partials and counters in the scratch; and within the parity bar of the oracle."""
    zha.get_status(clear=True)
    # another shape first: other batch, heads and cache length leave other contents behind
    other = _case(batch=1, Hkv=1, G=2, d=128, N=7000 + 13, seed_base=300)
    zha.route(other["cfg"], other["tree"], other["Qd"], other["N"], other["sel"], other["cnt"], other["ws"])
    _noalloc(other)

    c = _case(batch=2, Hkv=2, G=4, d=128, N=40000, seed_base=100)
    cfg = c["cfg"]
    zha.route(cfg, c["tree"], c["Qd"], c["N"], c["sel"], c["cnt"], c["ws"])
    O_ref = torch.zeros((cfg.batch, 1, cfg.Hq, cfg.d), dtype=torch.float32, device="cuda")
    zha.attend(cfg, c["Kd"], c["Vd"], c["tree"], c["Qd"], c["N"], c["sel"], c["cnt"], O_ref, c["ws"])
    torch.cuda.synchronize()
    ref = O_ref.cpu()
    for _ in range(2):
        got = _noalloc(c)
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref), float((got - ref).abs().max())
    # the oracle, attending over the GPU's own index sets of one (sequence, KV head) slice
    s, h = 1, 1
    ot = oracle_tree(c["K"][s, h], cfg.N_cap, cfg, c["qref"][h])
    hs = slice(h * cfg.G, (h + 1) * cfg.G)
    sel, cnt = c["sel"].cpu(), c["cnt"].cpu()
    rep = check_queries(cfg, ot, c["K"][s, h], c["V"][s, h], cfg.N_cap - 1, c["Q"][s, 0, hs].float(),
                        sel[s, 0, hs], cnt[s, 0, hs], got[s, 0, hs].numpy(), cfg.p, Report())
    rep.check()
    assert zha.get_status(clear=True) == 0


def test_attend_noalloc_refuses_configurations_beyond_its_scratch():
    cfg = zha.Config(d=128, Hq=32, Hkv=8, B=64, b=16, batch=4, N_cap=1 << 20, p=0.95)
    assert zha.workspace_bytes(cfg) > 16 << 20
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        zha.attend_noalloc(cfg, z, z, z, z, z, torch.zeros((1, 1, 1, 4), dtype=torch.int32, device="cuda"), z,
                           torch.zeros(4, device="cuda"))
    assert e.value.code == 6 and "static scratch" in str(e.value)
