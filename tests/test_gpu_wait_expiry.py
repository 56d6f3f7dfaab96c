"""The failure path of a bounded device wait, driven without faulting anything: the
tensor-core decode attention is run with its wait bound set to 0, so its first wait
on another warp's progress gives up.  The call must return, raise ZHA_ERR_TIMEOUT in
the device status, and leave the GPU usable: after the bound is restored and the
workspace re-initialised, the same call is correct against the oracle."""
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from tests.zha_parity import Report, check_queries, oracle_tree

pytestmark = pytest.mark.gpu


def test_wait_expiry_raises_timeout_and_the_next_call_is_correct():
    batch, Hkv, G, d, N = 2, 2, 4, 128, 30000 + 7
    dt = torch.bfloat16
    K = torch.zeros((batch, Hkv, N, d), dtype=dt)
    V = torch.zeros_like(K)
    Q = torch.zeros((batch, 1, G * Hkv, d), dtype=dt)
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice("test", 500 + s, h, N, d, 12, K[s, h], V[s, h], run=2048)
            Q[s, 0, h * G:(h + 1) * G] = W.cluster_queries("test", 500 + s, h, G, 1, cl)[0].to(dt)
    qref = W.reference_queries("test", Hkv, 1, d)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=N, p=0.95)
    assert zha.attend_kernel(cfg) == "attend_tc_kernel"   # the kernel whose waits the bound governs
    Kd, Vd, Qd = K.cuda(), V.cuda(), Q.cuda()
    Nt = torch.full((batch,), N, dtype=torch.int32, device="cuda")
    tree = zha.alloc_tree(cfg)
    ws = zha.alloc_workspace(cfg)
    sel = torch.zeros((batch, 1, G * Hkv, N // 64), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((batch, 1, G * Hkv), dtype=torch.int32, device="cuda")
    O = torch.zeros((batch, 1, G * Hkv, d), dtype=torch.float32, device="cuda")
    zha.get_status(clear=True)
    zha.build(cfg, Kd, qref.cuda(), Nt, tree)
    zha.route(cfg, tree, Qd, Nt, sel, cnt, ws)
    torch.cuda.synchronize()
    prev = zha.set_wait_limit(0)
    try:
        zha.attend(cfg, Kd, Vd, tree, Qd, Nt, None, None, O, ws)
        torch.cuda.synchronize()          # the call ended
    finally:
        zha.set_wait_limit(prev)
    bits = zha.get_status(clear=True)
    assert bits & (1 << 5), f"expected ZHA_ERR_TIMEOUT, status {zha.status_names(bits)}"
    # the context is intact: re-initialise the workspace and run again with the default bound
    zha.workspace_init(cfg, ws)
    O.fill_(float("nan"))
    zha.route(cfg, tree, Qd, Nt, sel, cnt, ws)
    zha.attend(cfg, Kd, Vd, tree, Qd, Nt, None, None, O, ws)
    torch.cuda.synchronize()
    assert zha.get_status(clear=True) == 0
    o, sl, ct = O.cpu(), sel.cpu(), cnt.cpu()
    rep = Report()
    for s in range(batch):
        for h in range(Hkv):
            ot = oracle_tree(K[s, h], N, cfg, qref[h])
            hs = slice(h * G, (h + 1) * G)
            check_queries(cfg, ot, K[s, h], V[s, h], N - 1, Q[s, 0, hs].float(), sl[s, 0, hs], ct[s, 0, hs],
                          o[s, 0, hs].numpy(), cfg.p, rep)
    rep.check()
