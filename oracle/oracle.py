"""ctypes glue around the fp64 C oracle (zha_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg use it; the library never does.  This file only
marshals arrays; every step of the method is in zha_oracle.c.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compiles zha_oracle.c into liboracle.so next to it (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_levels.argtypes = [I64, I32, I32, I32, P, I32]
        L.oracle_levels.restype = I32
        L.oracle_build.argtypes = [P, I32, I64, I32, I32, I32, I32, I32, P, D, P, P]
        L.oracle_build.restype = None
        L.oracle_route.argtypes = [P, I32, I32, I32, I32, I64, I32, P, P, D, P, P, P, P, P]
        L.oracle_route.restype = I64
        L.oracle_index_set.argtypes = [P, I64, I64, I32, I64, P]
        L.oracle_index_set.restype = I64
        L.oracle_attend.argtypes = [P, P, P, I32, I32, P, I64, D, P]
        L.oracle_attend.restype = None
        L.oracle_build_v.argtypes = [P, P, I32, I64, I32, I32, I32, I32, I32, P, D, P, P, P]
        L.oracle_build_v.restype = None
        L.oracle_route2.argtypes = [P, I32, I32, I32, I32, I64, I32, P, P, D, P, P, P, P, P, P, P, P, P]
        L.oracle_route2.restype = I64
        L.oracle_attend_vsum.argtypes = [P, P, P, I32, I32, P, I64, D, P, P, I64, P]
        L.oracle_attend_vsum.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _kv_array(x) -> tuple[np.ndarray, int]:
    """Host array of keys/values and its dtype code: 0 = fp32, 1 = bf16 bits."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), 1
            return x.to(torch.float32).numpy(), 0
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, 1
    return np.ascontiguousarray(x, dtype=np.float32), 0


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float64)


def levels(N: int, B: int, b: int, L_fixed: int = 0) -> list[int]:
    """Nodes per level (level 1 first); L_fixed > 0 fixes the depth."""
    n = np.zeros(64, dtype=np.int64)
    L = lib().oracle_levels(N, B, b, L_fixed, _ptr(n), 64)
    if L < 0:
        raise ValueError("too many levels")
    return [int(v) for v in n[:L]]


@dataclass
class Tree:
    N: int
    B: int
    b: int
    R: int
    d: int
    n: list            # nodes per level, level 1 first
    khat: np.ndarray   # [total nodes][R][d] float64, level 1 first
    bhat: np.ndarray   # [total nodes][R]
    scale: float
    vhat: np.ndarray | None = None   # [total nodes][R][d] value summaries, when built with V

    @property
    def L(self) -> int:
        return len(self.n)

    def level(self, l: int) -> tuple[np.ndarray, np.ndarray]:
        off = sum(self.n[:l - 1])
        return self.khat[off:off + self.n[l - 1]], self.bhat[off:off + self.n[l - 1]]


def build_tree(K_slice, N: int, B: int, b: int, qref_slice, scale: float | None = None,
               L_fixed: int = 0, V_slice=None) -> Tree:
    """K_slice: [>= N, d] keys of one (sequence, KV head); qref_slice: [>= L][R][d].
    With V_slice, the value summaries too (Tree.vhat)."""
    K, dt = _kv_array(K_slice)
    d = K.shape[-1]
    n = levels(N, B, b, L_fixed)
    q = _f64(qref_slice)
    R = q.shape[1]
    q = np.ascontiguousarray(q[:len(n)])
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    tot = sum(n)
    khat = np.zeros((max(tot, 1), R, d), dtype=np.float64)
    bhat = np.zeros((max(tot, 1), R), dtype=np.float64)
    if V_slice is None:
        lib().oracle_build(_ptr(K), dt, N, d, B, b, R, len(n), _ptr(q), scale, _ptr(khat), _ptr(bhat))
        return Tree(N, B, b, R, d, n, khat[:tot], bhat[:tot], scale)
    V, dv = _kv_array(V_slice)
    assert dv == dt
    vhat = np.zeros_like(khat)
    lib().oracle_build_v(_ptr(K), _ptr(V), dt, N, d, B, b, R, len(n), _ptr(q), scale, _ptr(khat), _ptr(bhat),
                         _ptr(vhat))
    return Tree(N, B, b, R, d, n, khat[:tot], bhat[:tot], scale, vhat[:tot])


@dataclass
class Route:
    sel: np.ndarray      # kept level-1 block ids, ascending
    n_cand: np.ndarray   # per level (level 1 first)
    n_kept: np.ndarray
    margin: np.ndarray
    pr_node: np.ndarray | None = None    # pruned nodes (global index, level 1 first), their planes
    pr_plane: np.ndarray | None = None   # and scores, level by level from the top
    pr_s: np.ndarray | None = None

    @property
    def min_margin(self) -> float:
        return float(self.margin.min()) if len(self.margin) else math.inf


def route(q, tree: Tree, p) -> Route:
    """Routes one query vector q [d] through the tree; p is a float or per-level list."""
    qd = _f64(q).reshape(-1)
    L = tree.L
    pl = np.asarray([p] * L if np.isscalar(p) else list(p)[:L], dtype=np.float64)
    sel = np.zeros(max(tree.n[0], 1), dtype=np.int64)
    nc = np.zeros(L, dtype=np.int64)
    nk = np.zeros(L, dtype=np.int64)
    mg = np.zeros(L, dtype=np.float64)
    kh = tree.khat if tree.khat.size else np.zeros((1, tree.R, tree.d))
    bh = tree.bhat if tree.bhat.size else np.zeros((1, tree.R))
    tot = max(sum(tree.n), 1)
    prn = np.zeros(tot, dtype=np.int64)
    prp = np.zeros(tot, dtype=np.int32)
    prs = np.zeros(tot, dtype=np.float64)
    npr = np.zeros(1, dtype=np.int64)
    cnt = lib().oracle_route2(_ptr(qd), tree.d, tree.R, tree.B, tree.b, tree.N, L, _ptr(kh), _ptr(bh),
                              tree.scale, _ptr(pl), _ptr(sel), _ptr(nc), _ptr(nk), _ptr(mg),
                              _ptr(prn), _ptr(prp), _ptr(prs), _ptr(npr))
    k = int(npr[0])
    return Route(sel[:cnt].copy(), nc, nk, mg, prn[:k].copy(), prp[:k].copy(), prs[:k].copy())


def index_set(sel, t: int, B: int, n1: int) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int64))
    out = np.zeros(t + 1, dtype=np.int64)
    c = lib().oracle_index_set(_ptr(s) if len(s) else None, len(s), t, B, n1, _ptr(out))
    return out[:c].copy()


def attend(q, K_slice, V_slice, idx, scale: float | None = None) -> np.ndarray:
    qd = _f64(q).reshape(-1)
    K, dt = _kv_array(K_slice)
    V, dt2 = _kv_array(V_slice)
    assert dt == dt2
    d = K.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int64))
    o = np.zeros(d, dtype=np.float64)
    lib().oracle_attend(_ptr(qd), _ptr(K), _ptr(V), dt, d, _ptr(ix), len(ix), scale, _ptr(o))
    return o


def dense(q, K_slice, V_slice, t: int, scale: float | None = None) -> np.ndarray:
    """Full causal attention of a query at position t over keys [0, t]."""
    return attend(q, K_slice, V_slice, np.arange(t + 1, dtype=np.int64), scale)


def decode_query(q, tree: Tree, K_slice, V_slice, t: int, p) -> tuple[Route, np.ndarray, np.ndarray]:
    """Route, index set and attention of one query at position t: (route, idx, o)."""
    r = route(q, tree, p)
    idx = index_set(r.sel, t, tree.B, tree.n[0])
    return r, idx, attend(q, K_slice, V_slice, idx, tree.scale)


def attend_vsum(q, K_slice, V_slice, idx, tree: Tree, rt: Route) -> np.ndarray:
    """Attention over idx plus the pruned nodes of rt as pseudo-keys (score, value summary)."""
    assert tree.vhat is not None, "the tree was built without V"
    qd = _f64(q).reshape(-1)
    K, dt = _kv_array(K_slice)
    V, dt2 = _kv_array(V_slice)
    assert dt == dt2
    d = K.shape[-1]
    ix = np.ascontiguousarray(np.asarray(idx, dtype=np.int64))
    prv = np.ascontiguousarray(tree.vhat[rt.pr_node, rt.pr_plane].reshape(-1, d)) if len(rt.pr_node) \
        else np.zeros((1, d))
    prs = np.ascontiguousarray(rt.pr_s, dtype=np.float64) if len(rt.pr_s) else np.zeros(1)
    o = np.zeros(d, dtype=np.float64)
    lib().oracle_attend_vsum(_ptr(qd), _ptr(K), _ptr(V), dt, d, _ptr(ix), len(ix), tree.scale,
                             _ptr(prs), _ptr(prv), len(rt.pr_node), _ptr(o))
    return o


def decode_query_vsum(q, tree: Tree, K_slice, V_slice, t: int, p) -> tuple[Route, np.ndarray, np.ndarray]:
    """decode_query with the pruned subtrees' value summaries: (route, idx, o)."""
    r = route(q, tree, p)
    idx = index_set(r.sel, t, tree.B, tree.n[0])
    return r, idx, attend_vsum(q, K_slice, V_slice, idx, tree, r)
