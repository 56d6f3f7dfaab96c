"""zha_extend: growing a tree over keys already written into the cache (a
prefill chunk, a batch of tokens) gives, bit for bit, the tree zha_build makes
at the new length ("Zyphra Hierarchical Attention: The End of Quadratic
Attention?", the tree is built on the fly as the context grows)."""
import pytest
import torch

from hierarchical_tree_indexed_b200 import workloads as W
from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O
from tests.zha_parity import Decoder, assert_status_clean

pytestmark = pytest.mark.gpu


def keys(batch, Hkv, N, d, R, L_fixed=0):
    K = torch.zeros((batch, Hkv, N, d), dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    for s in range(batch):
        for h in range(Hkv):
            W.fill_planted_slice("test", s, h, N, d, 3, K[s, h], V[s, h], run=min(300, N // 4))
    return K, V, W.reference_queries("test", Hkv, R, d)


@pytest.mark.parametrize("B,b,R,L_fixed", [(16, 4, 1, 0), (16, 4, 2, 0), (8, 8, 1, 4)])
def test_extend_matches_rebuild_bitwise(B, b, R, L_fixed):
    batch, Hkv, d = 2, 2, 64
    N_cap = 6000
    K, V, qref = keys(batch, Hkv, N_cap, d, R, L_fixed)
    cfg = zha.Config(d=d, Hq=Hkv, Hkv=Hkv, B=B, b=b, batch=batch, N_cap=N_cap, p=0.9, R=R, L_fixed=L_fixed)
    Kd = K.cuda()
    grow = Decoder(cfg, Kd, V.cuda(), qref.cuda(), [0, 37])
    grow.build()
    ref = Decoder(cfg, Kd, V.cuda(), qref.cuda(), [0, 37])
    n = [0, 37]
    # chunks of every shape: one key, part of a block, a block, across blocks, many blocks,
    # growth of the depth; the two sequences grow differently
    for step, (a, c) in enumerate([(1, 0), (15, 27), (16, 16), (17, 1), (200, 64), (1000, 333), (0, 2000),
                                   (3000, 5), (1, 1)]):
        n = [n[0] + a, n[1] + c]
        N = torch.tensor(n, dtype=torch.int32, device="cuda")
        zha.extend(cfg, Kd, N, grow.tree)
        ref.N.copy_(N)
        ref.tree.zero_()
        ref.build()
        torch.cuda.synchronize()
        assert zha.tree_count_view(cfg, grow.tree).cpu().tolist() == n
        for s in range(batch):
            lv = O.levels(n[s], B, b, L_fixed)
            for l in range(1, len(lv) + 1):
                ka, ba = zha.tree_level_view(cfg, grow.tree, l)
                kb, bb = zha.tree_level_view(cfg, ref.tree, l)
                m = lv[l - 1]
                assert torch.equal(ka[s, :, :m], kb[s, :, :m]), (step, s, l)
                assert torch.equal(ba[s, :, :m], bb[s, :, :m]), (step, s, l)
    assert_status_clean()


def test_extend_refuses_to_shrink():
    batch, Hkv, d, B, b = 1, 1, 64, 16, 4
    K, V, qref = keys(batch, Hkv, 2000, d, 1)
    cfg = zha.Config(d=d, Hq=1, Hkv=1, B=B, b=b, batch=batch, N_cap=2000, p=0.9)
    dec = Decoder(cfg, K.cuda(), V.cuda(), qref.cuda(), [1000])
    dec.build()
    zha.get_status(clear=True)
    zha.extend(cfg, dec.K, torch.tensor([900], dtype=torch.int32, device="cuda"), dec.tree)
    bits = zha.get_status(clear=True)
    assert bits & (1 << 1), zha.status_names(bits)
    assert zha.tree_count_view(cfg, dec.tree).cpu().tolist() == [1000]
