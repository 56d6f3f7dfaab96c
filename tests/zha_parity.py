"""Shared helpers of the parity tests: run the CUDA path through the C ABI and
check it against the fp64 oracle, slice by slice.

Bars (from the workload definitions):
  * index sets: bit-exact wherever the oracle's cut margin > 1e-4;
  * outputs: fp32 mode max|d| <= 1e-3; bf16 mode ||d||_inf <= 2e-2 ||o||_inf per (query, head),
    both against the oracle's own set and against the oracle attending over the
    GPU's set (the second also at a tight 1e-3 relative bound, which a dropped or
    doubled key would break).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from hierarchical_tree_indexed_b200 import zha
from oracle import oracle as O

MARGIN = 1e-4
TOL_F32 = 1e-3
TOL_BF16_REL = 2e-2
TOL_TIGHT_REL = 1e-3
SUMMARY_ATOL = 2e-4


@dataclass
class Report:
    queries: int = 0
    exact_required: int = 0
    mismatches_required: int = 0
    mismatches_low_margin: int = 0
    low_margin: int = 0
    excused: int = 0                # margin > 1e-4, but the walk met a node the caller excused
    max_err_own: float = 0.0        # vs the oracle over the oracle's set (relative in bf16)
    max_err_gpu_set: float = 0.0    # vs the oracle over the GPU's set
    read_keys: list = field(default_factory=list)

    def check(self):
        assert self.mismatches_required == 0, f"{self.mismatches_required} index sets differ beyond the margin"

    def summary(self) -> dict:
        """The counts the parity bar is stated in: index sets required bit-exact (margin > 1e-4) and
        how many of them differ, and the same for the queries below the margin (reported only)."""
        return {"queries": self.queries, "exact_required": self.exact_required,
                "mismatches_required": self.mismatches_required, "low_margin": self.low_margin,
                "mismatches_low_margin": self.mismatches_low_margin, "excused": self.excused,
                "max_err_gpu_set": self.max_err_gpu_set, "max_err_own": self.max_err_own}


def oracle_tree(K_slice_cpu, N, cfg: zha.Config, qref_slice):
    return O.build_tree(K_slice_cpu, N, cfg.B, cfg.b, qref_slice, scale=cfg.softmax_scale, L_fixed=cfg.L_fixed)


def compare_tree(cfg: zha.Config, tree: torch.Tensor, ot: O.Tree, s: int, h: int, atol=SUMMARY_ATOL):
    """GPU summaries of slice (s, h) against the oracle's, every level and node."""
    for l in range(1, ot.L + 1):
        kh, bh = zha.tree_level_view(cfg, tree, l)
        n = ot.n[l - 1]
        if n == 0:
            continue
        g_k = kh[s, h, :n].double().cpu().numpy()        # [n][R][d], every plane
        g_b = bh[s, h, :n].double().cpu().numpy()
        o_k, o_b = ot.level(l)
        dk = np.max(np.abs(g_k - o_k))
        db = np.max(np.abs(g_b - o_b))
        assert dk <= atol and db <= atol, f"level {l}: khat err {dk:.3g}, bhat err {db:.3g}"


def out_err(o_gpu: np.ndarray, o_ref: np.ndarray, dtype: str) -> float:
    d = float(np.max(np.abs(o_gpu - o_ref)))
    return d if dtype == "f32" else d / max(float(np.max(np.abs(o_ref))), 1e-30)


def check_queries(cfg: zha.Config, ot: O.Tree, K_slice, V_slice, t, queries, sel_rows, counts, outs,
                  p, rep: Report, tight_of_v: float | None = None, excuse=None):
    """queries: [nq][d] (CPU tensors, the exact values the GPU read); sel_rows/counts/outs: GPU results.
    t: the queries' position, or one position per query.  tight_of_v: when given, the tight check
    against the oracle over the GPU's set is |d|_inf <= tight_of_v * max |v| over that set (the
    tensor-core path rounds the softmax weights to bf16 before P V) instead of 1e-3 of |o|_inf.
    excuse: when given, excuse(route) -> True lifts the exactness requirement of a query whose
    oracle walk scored a node the caller cannot compare (counted in rep.excused)."""
    bar = TOL_F32 if cfg.dtype == "f32" else TOL_BF16_REL
    for i in range(len(queries)):
        q = queries[i]
        ti = t if isinstance(t, (int, np.integer)) else int(t[i])
        rt = O.route(q, ot, p)
        g_sel = np.asarray(sel_rows[i][:counts[i]], dtype=np.int64)
        rep.queries += 1
        same = len(g_sel) == len(rt.sel) and np.array_equal(g_sel, rt.sel)
        if rt.min_margin > MARGIN and excuse is not None and excuse(rt):
            rep.excused += 1
        elif rt.min_margin > MARGIN:
            rep.exact_required += 1
            rep.mismatches_required += 0 if same else 1
        else:
            rep.low_margin += 1
            rep.mismatches_low_margin += 0 if same else 1
        o_g = np.asarray(outs[i], dtype=np.float64)
        idx_g = O.index_set(g_sel, ti, cfg.B, ot.n[0])
        rep.read_keys.append(len(idx_g))
        o_gset = O.attend(q, K_slice, V_slice, idx_g, ot.scale)
        e2 = out_err(o_g, o_gset, cfg.dtype)
        rep.max_err_gpu_set = max(rep.max_err_gpu_set, e2)
        assert e2 <= bar, f"query {i}: output error {e2:.3g} against the oracle over the GPU's set"
        if tight_of_v is None:
            tight = float(np.max(np.abs(o_g - o_gset))) / max(float(np.max(np.abs(o_gset))), 1e-30)
            assert tight <= TOL_TIGHT_REL, f"query {i}: relative error {tight:.3g} over the GPU's set"
        else:
            vmax = float(np.max(np.abs(np.asarray(V_slice[torch.as_tensor(idx_g)].float()))))
            tight = float(np.max(np.abs(o_g - o_gset))) / vmax
            assert tight <= tight_of_v, f"query {i}: error {tight:.3g} of max|v| over the GPU's set"
        if same:
            rep.max_err_own = max(rep.max_err_own, e2)
        else:
            idx_o = O.index_set(rt.sel, ti, cfg.B, ot.n[0])
            o_own = O.attend(q, K_slice, V_slice, idx_o, ot.scale)
            rep.max_err_own = max(rep.max_err_own, out_err(o_g, o_own, cfg.dtype))
    return rep


class Decoder:
    """Device buffers of one configuration, driven through the C ABI."""

    def __init__(self, cfg: zha.Config, K: torch.Tensor, V: torch.Tensor, qref: torch.Tensor, N: list[int]):
        self.cfg = cfg
        self.K, self.V = K, V
        self.qref = qref
        self.N = torch.tensor(N, dtype=torch.int32, device="cuda")
        self.tree = zha.alloc_tree(cfg)
        self.ws = zha.alloc_workspace(cfg)
        n1cap = max(cfg.N_cap // cfg.B, 1)
        self.sel = torch.zeros((cfg.batch, 1, cfg.Hq, n1cap), dtype=torch.int32, device="cuda")
        self.cnt = torch.zeros((cfg.batch, 1, cfg.Hq), dtype=torch.int32, device="cuda")
        self.O = torch.zeros((cfg.batch, 1, cfg.Hq, cfg.d), dtype=torch.float32, device="cuda")

    def build(self):
        self._q = zha.build(self.cfg, self.K, self.qref, self.N, self.tree, V=self.V)

    def route_attend(self, Q: torch.Tensor):
        zha.route(self.cfg, self.tree, Q, self.N, self.sel, self.cnt, self.ws)
        zha.attend(self.cfg, self.K, self.V, self.tree, Q, self.N, self.sel, self.cnt, self.O, self.ws)

    def decode(self, q, k_new, v_new):
        zha.decode(self.cfg, self.K, self.V, self.tree, q, k_new, v_new, self.N, self.O, self.ws)

    def dense(self, Q):
        zha.dense(self.cfg, self.K, self.V, Q, self.N, self.O, self.ws)

    def results(self):
        torch.cuda.synchronize()
        return self.sel.cpu(), self.cnt.cpu(), self.O.cpu()


def assert_status_clean():
    bits = zha.get_status(clear=True)
    assert bits == 0, f"device status raised: {zha.status_names(bits)}"
