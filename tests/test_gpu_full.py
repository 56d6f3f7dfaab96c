"""The 1M-token decode workload at full size (batch 4, 32 query / 8 KV heads,
d = 128, bf16), in the launch configuration the benchmark times, checked on
sampled (sequence, KV head) slices against the oracle."""
import numpy as np
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O
from tests.zha_parity import Report, assert_status_clean, check_queries, compare_tree, oracle_tree

pytestmark = pytest.mark.gpu

SAMPLES = [(0, 0), (3, 7)]


def test_decode_1m_full_size_sampled():
    w = W.WORKLOADS["decode1m"]
    steps = 2
    N_cap = w.N + steps
    data = W.planted(w, device="cuda", N_cap=N_cap, n_queries=steps)
    K, V, Q = data["K"], data["V"], data["Q"]
    kn, vn = data["k_new"], data["v_new"]
    torch.cuda.synchronize()
    host = {sh: (K[sh].cpu().clone(), V[sh].cpu().clone()) for sh in SAMPLES}   # generator output
    for sh in SAMPLES:
        for i in range(steps):
            host[sh][0][w.N + i] = kn[i, sh[0], sh[1]].cpu()
            host[sh][1][w.N + i] = vn[i, sh[0], sh[1]].cpu()
    Qh, qref = Q.cpu(), data["qref"].cpu()
    cfg = zha.Config(d=w.d, Hq=w.Hq, Hkv=w.Hkv, B=w.B, b=w.b, batch=w.batch, N_cap=N_cap, p=w.p)
    N = torch.full((w.batch,), w.N, dtype=torch.int32, device="cuda")
    tree = zha.alloc_tree(cfg)
    ws = zha.alloc_workspace(cfg)
    O_ = torch.zeros((w.batch, 1, w.Hq, w.d), dtype=torch.float32, device="cuda")
    zha.get_status(clear=True)
    zha.build(cfg, K, data["qref"], N, tree)
    rep = Report()
    for i in range(steps):
        zha.decode(cfg, K, V, tree, Q[i].reshape(w.batch, 1, w.Hq, w.d).contiguous(), kn[i].contiguous(),
                   vn[i].contiguous(), N, O_, ws)
        torch.cuda.synchronize()
        n_now = w.N + i + 1
        sel = ws  # noqa: F841  (selection stays in the workspace)
        o = O_.cpu()
        for (s, h) in SAMPLES:
            Kh, Vh = host[(s, h)]
            ot = oracle_tree(Kh, n_now, cfg, qref[h])
            if i == steps - 1:
                compare_tree(cfg, tree, ot, s, h)
            for g in range(w.G):
                hq = h * w.G + g
                q = Qh[i, s, hq]
                rt = O.route(q, ot, w.p)
                rep.queries += 1
                if rt.min_margin <= 1e-4:
                    rep.low_margin += 1
                    continue
                rep.exact_required += 1
                idx = O.index_set(rt.sel, n_now - 1, w.B, ot.n[0])
                ref = O.attend(q, Kh, Vh, idx)
                rel = float(np.max(np.abs(o[s, 0, hq].numpy() - ref)) / np.max(np.abs(ref)))
                assert rel <= 1e-3, (i, s, hq, rel)
                rep.read_keys.append(len(idx))
    assert rep.exact_required >= rep.queries // 2, rep
    assert_status_clean()
    print(f"1M sampled: {rep.exact_required}/{rep.queries} checked, mean keys read per head "
          f"{np.mean(rep.read_keys):.0f} ({np.mean(rep.read_keys) / w.N * 100:.2f}% of the cache)")
