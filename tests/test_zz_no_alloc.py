"""zha_attend_noalloc, the attention entry point for callers that cannot
allocate device memory (it runs on the library's static device scratch
instead of a caller-provided workspace), against zha_attend with a workspace.

Collected last on purpose: the static scratch keeps whatever the previous call
left, so this file also checks that results do not depend on what ran before.
"""
import ctypes

import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha

pytestmark = pytest.mark.gpu

TOL_BF16_REL = 2e-2      # the bf16 output bar of the parity tests


def _inputs(batch, Hkv, G, d, N):
    dt = torch.bfloat16
    K = torch.zeros((batch, Hkv, N, d), dtype=dt)
    V = torch.zeros_like(K)
    Q = torch.zeros((batch, 1, G * Hkv, d), dtype=dt)
    for s in range(batch):
        for h in range(Hkv):
            cl = W.fill_planted_slice("test", 100 + s, h, N, d, 16, K[s, h], V[s, h], run=N // 8)
            Q[s, 0, h * G:(h + 1) * G] = W.cluster_queries("test", 100 + s, h, G, 1, cl)[0].to(dt)
    return K.cuda(), V.cuda(), Q.cuda(), W.reference_queries("test", Hkv, 1, d).cuda()


def test_attend_noalloc_matches_attend_twice_in_a_row():
    batch, Hkv, G, d, N = 2, 2, 4, 128, 40000
    K, V, Q, qref = _inputs(batch, Hkv, G, d, N)
    cfg = zha.Config(d=d, Hq=G * Hkv, Hkv=Hkv, B=64, b=16, batch=batch, N_cap=N, p=0.95)
    Nt = torch.full((batch,), N, dtype=torch.int32, device="cuda")
    tree = zha.alloc_tree(cfg)
    ws = zha.alloc_workspace(cfg)
    sel = torch.zeros((batch, 1, G * Hkv, N // 64), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((batch, 1, G * Hkv), dtype=torch.int32, device="cuda")
    zha.get_status(clear=True)
    zha.build(cfg, K, qref, Nt, tree)
    zha.route(cfg, tree, Q, Nt, sel, cnt, ws)
    O_ref = torch.zeros((batch, 1, G * Hkv, d), dtype=torch.float32, device="cuda")
    zha.attend(cfg, K, V, tree, Q, Nt, sel, cnt, O_ref, ws)
    torch.cuda.synchronize()
    ref = O_ref.cpu().numpy()
    for _ in range(2):
        O = torch.full_like(O_ref, float("nan"))
        zha.attend_noalloc(cfg, K, V, tree, Q, Nt, sel, cnt, O)
        torch.cuda.synchronize()
        got = O.cpu().numpy()
        assert np.isfinite(got).all()
        for s in range(batch):
            for h in range(G * Hkv):
                err = np.max(np.abs(got[s, 0, h] - ref[s, 0, h])) / np.max(np.abs(ref[s, 0, h]))
                assert err <= TOL_BF16_REL, (s, h, err)
    assert zha.get_status(clear=True) == 0


def test_attend_noalloc_refuses_configurations_beyond_its_scratch():
    cfg = zha.Config(d=128, Hq=32, Hkv=8, B=64, b=16, batch=4, N_cap=1 << 20, p=0.95)
    assert zha.workspace_bytes(cfg) > 16 << 20
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(zha.ZhaError) as e:
        zha.attend_noalloc(cfg, z, z, z, z, z, torch.zeros((1, 1, 1, 4), dtype=torch.int32, device="cuda"), z,
                           torch.zeros(4, device="cuda"))
    assert e.value.code == 6 and "static scratch" in str(e.value)
