"""ctypes binding of the C ABI in include/zha.h (libzha.so, built for sm_100a).

Argument marshalling only: torch tensors are passed as device pointers and the
current CUDA stream as the stream handle; every step of the path runs in the
library's kernels.  There is no fallback: if libzha.so is missing or cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

MAX_LEVELS = 16
F32, BF16 = 0, 1
STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CAPACITY", 4: "CUDA", 5: "TIMEOUT",
          6: "WORKSPACE"}

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzha.so")
_lib = None


class ZhaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"zha error {code} ({STATUS.get(code, '?')}): {msg}")
        self.code = code


class ZhaConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("B", ctypes.c_int32), ("b", ctypes.c_int32), ("R", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("batch", ctypes.c_int32), ("N_cap", ctypes.c_int64),
                ("L_fixed", ctypes.c_int32), ("scale", ctypes.c_float),
                ("p", ctypes.c_float * MAX_LEVELS), ("vsum", ctypes.c_int32)]


EXPORTS = ["zha_levels_cap", "zha_tree_bytes", "zha_tree_level", "zha_tree_level_v", "zha_tree_count_offset", "zha_workspace_bytes", "zha_workspace_init", "zha_workspace_stats", "zha_attend_kernel", "zha_build",
           "zha_extend", "zha_append", "zha_route", "zha_attend", "zha_attend_noalloc", "zha_decode", "zha_dense", "zha_get_status",
           "zha_set_wait_limit", "zha_last_error"]


def lib():
    """Loads libzha.so (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m hierarchical_tree_indexed_b200.build_lib`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    C = ctypes.POINTER(ZhaConfig)
    sig = {
        "zha_levels_cap": [C, P],
        "zha_tree_bytes": [C, P],
        "zha_tree_level": [C, I32, P, P, P],
        "zha_tree_level_v": [C, I32, P],
        "zha_tree_count_offset": [C, P],
        "zha_workspace_bytes": [C, I32, P],
        "zha_workspace_init": [C, P, SZ, P],
        "zha_workspace_stats": [C, I32, P, P, P],
        "zha_attend_kernel": [C, I32, P],
        "zha_build": [C, P, P, P, P, P, P],
        "zha_extend": [C, P, P, P, P, P],
        "zha_append": [C, P, P, P, P, P, P, P],
        "zha_route": [C, P, P, I32, P, P, P, I32, P, SZ, P],
        "zha_attend": [C, P, P, P, P, I32, P, P, P, I32, P, P, SZ, P],
        "zha_attend_noalloc": [C, P, P, P, P, I32, P, P, P, I32, P, P],
        "zha_decode": [C, P, P, P, P, P, P, P, P, P, SZ, P],
        "zha_dense": [C, P, P, P, I32, P, P, P, SZ, P],
        "zha_get_status": [P, I32, P],
        "zha_set_wait_limit": [ctypes.c_uint64, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.zha_last_error.argtypes = []
    L.zha_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _check(rc: int):
    if rc != 0:
        raise ZhaError(rc, lib().zha_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors passed to the library must be contiguous")
        return t.data_ptr()
    return int(t)


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


@dataclass
class Config:
    """Python mirror of zha_config (see include/zha.h)."""
    d: int
    Hq: int
    Hkv: int
    B: int
    b: int
    batch: int
    N_cap: int
    dtype: str = "bf16"
    p: float | list = 0.95
    R: int = 1
    L_fixed: int = 0
    scale: float = 0.0
    vsum: int = 0

    def c(self) -> ZhaConfig:
        cfg = ZhaConfig()
        cfg.d, cfg.Hq, cfg.Hkv, cfg.B, cfg.b, cfg.R = self.d, self.Hq, self.Hkv, self.B, self.b, self.R
        cfg.dtype = {"f32": F32, "bf16": BF16}[self.dtype]
        cfg.batch, cfg.N_cap, cfg.L_fixed, cfg.scale = self.batch, self.N_cap, self.L_fixed, self.scale
        cfg.vsum = self.vsum
        ps = [self.p] * MAX_LEVELS if isinstance(self.p, (int, float)) else list(self.p)
        ps = ps + [ps[-1]] * (MAX_LEVELS - len(ps))
        for i in range(MAX_LEVELS):
            cfg.p[i] = float(ps[i])
        return cfg

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)


def levels_cap(cfg: Config) -> int:
    v = ctypes.c_int32()
    _check(lib().zha_levels_cap(ctypes.byref(cfg.c()), ctypes.byref(v)))
    return v.value


def tree_bytes(cfg: Config) -> int:
    v = ctypes.c_size_t()
    _check(lib().zha_tree_bytes(ctypes.byref(cfg.c()), ctypes.byref(v)))
    return v.value


def tree_level_view(cfg: Config, tree: torch.Tensor, level: int) -> tuple[torch.Tensor, torch.Tensor]:
    """(khat [batch][Hkv][nodes_cap][R][d], bhat [batch][Hkv][nodes_cap][R]) fp32 views of one level."""
    ko, bo, nc = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int64()
    _check(lib().zha_tree_level(ctypes.byref(cfg.c()), level, ctypes.byref(ko), ctypes.byref(bo), ctypes.byref(nc)))
    n = nc.value
    kh = tree[ko.value:ko.value + 4 * cfg.batch * cfg.Hkv * n * cfg.R * cfg.d].view(torch.float32)
    bh = tree[bo.value:bo.value + 4 * cfg.batch * cfg.Hkv * n * cfg.R].view(torch.float32)
    return kh.view(cfg.batch, cfg.Hkv, n, cfg.R, cfg.d), bh.view(cfg.batch, cfg.Hkv, n, cfg.R)


def tree_vhat_view(cfg: Config, tree: torch.Tensor, level: int) -> torch.Tensor:
    """vhat [batch][Hkv][nodes_cap][d] fp32 view of one level (cfg.vsum = 1)."""
    vo, ko, bo, nc = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int64()
    _check(lib().zha_tree_level(ctypes.byref(cfg.c()), level, ctypes.byref(ko), ctypes.byref(bo), ctypes.byref(nc)))
    _check(lib().zha_tree_level_v(ctypes.byref(cfg.c()), level, ctypes.byref(vo)))
    n = nc.value
    vh = tree[vo.value:vo.value + 4 * cfg.batch * cfg.Hkv * n * cfg.d].view(torch.float32)
    return vh.view(cfg.batch, cfg.Hkv, n, cfg.d)


def tree_count_view(cfg: Config, tree: torch.Tensor) -> torch.Tensor:
    o = ctypes.c_size_t()
    _check(lib().zha_tree_count_offset(ctypes.byref(cfg.c()), ctypes.byref(o)))
    return tree[o.value:o.value + 4 * cfg.batch].view(torch.int32)


def workspace_bytes(cfg: Config, n_q: int = 1) -> int:
    v = ctypes.c_size_t()
    _check(lib().zha_workspace_bytes(ctypes.byref(cfg.c()), n_q, ctypes.byref(v)))
    return v.value


def workspace_stats_view(cfg: Config, ws: torch.Tensor, n_q: int = 1):
    """int32 views (rows [batch*Hkv] keys gathered per group, cand [batch*n_q*Hq] nodes scored per
    query head, scanned [batch*Hkv] distinct nodes the route read per group; with n_q > 1 scanned
    is cand)."""
    ro, co, so = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().zha_workspace_stats(ctypes.byref(cfg.c()), n_q, ctypes.byref(ro), ctypes.byref(co),
                                     ctypes.byref(so)))
    g, c = cfg.batch * cfg.Hkv, cfg.batch * n_q * cfg.Hq
    sn = c if n_q > 1 else g
    return (ws[ro.value:ro.value + 4 * g].view(torch.int32), ws[co.value:co.value + 4 * c].view(torch.int32),
            ws[so.value:so.value + 4 * sn].view(torch.int32))


def alloc_tree(cfg: Config, device="cuda") -> torch.Tensor:
    return torch.zeros(tree_bytes(cfg), dtype=torch.uint8, device=device)


ATTEND_KERNELS = ("attend_kernel", "attend_tc_kernel", "attend_prefill_kernel")


def attend_kernel(cfg: Config, n_q: int = 1) -> str:
    """Name of the attention kernel zha_attend runs for this configuration on the current device."""
    k = ctypes.c_int32()
    _check(lib().zha_attend_kernel(ctypes.byref(cfg.c()), n_q, ctypes.byref(k)))
    return ATTEND_KERNELS[k.value]


def alloc_workspace(cfg: Config, n_q: int = 1, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(workspace_bytes(cfg, n_q), dtype=torch.uint8, device=device)
    workspace_init(cfg, ws, stream)
    return ws


def workspace_init(cfg: Config, ws: torch.Tensor, stream=None):
    """Zeroes a workspace (after allocation, or after a call that raised ZHA_ERR_TIMEOUT)."""
    _check(lib().zha_workspace_init(ctypes.byref(cfg.c()), _ptr(ws), ws.numel(), _stream(stream)))


def build(cfg: Config, K, qref, N, tree, stream=None, V=None):
    """qref: [Hkv][>= levels_cap][R][d] fp32 (sliced to levels_cap here).  V: the value cache
    (read with cfg.vsum = 1)."""
    Lc = levels_cap(cfg)
    q = qref[:, :Lc].contiguous()
    _check(lib().zha_build(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(q), _ptr(N), _ptr(tree), _stream(stream)))
    return q   # keep alive until the copy has run


def extend(cfg: Config, K, N, tree, stream=None, V=None):
    """Grows the tree to index keys [0, N[s]) already written into K (see include/zha.h)."""
    _check(lib().zha_extend(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(N), _ptr(tree), _stream(stream)))


def append(cfg: Config, K, V, k_new, v_new, N, tree, stream=None):
    _check(lib().zha_append(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(k_new), _ptr(v_new), _ptr(N),
                            _ptr(tree), _stream(stream)))


def route(cfg: Config, tree, Q, N, sel, sel_count, ws, n_q: int = 1, stream=None):
    _check(lib().zha_route(ctypes.byref(cfg.c()), _ptr(tree), _ptr(Q), n_q, _ptr(N), _ptr(sel), _ptr(sel_count),
                           sel.shape[-1], _ptr(ws), ws.numel(), _stream(stream)))


def attend(cfg: Config, K, V, tree, Q, N, sel, sel_count, O, ws, n_q: int = 1, stream=None):
    """sel = sel_count = None: use the gather plan the last route() left in ws."""
    sel_cap = sel.shape[-1] if sel is not None else 0
    _check(lib().zha_attend(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(tree), _ptr(Q), n_q, _ptr(N), _ptr(sel),
                            _ptr(sel_count), sel_cap, _ptr(O), _ptr(ws), ws.numel(), _stream(stream)))


def attend_noalloc(cfg: Config, K, V, tree, Q, N, sel, sel_count, O, stream=None, n_q: int = 1):
    """zha_attend of decode queries (n_q = 1) without a workspace: the library's static device
    scratch (see include/zha.h).  n_q is passed through only so that a caller can see the
    library's own refusal of a chunked prefill."""
    _check(lib().zha_attend_noalloc(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(tree), _ptr(Q), n_q, _ptr(N),
                                    _ptr(sel), _ptr(sel_count), sel.shape[-1], _ptr(O), _stream(stream)))


def decode(cfg: Config, K, V, tree, q, k_new, v_new, N, O, ws, stream=None):
    _check(lib().zha_decode(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(tree), _ptr(q), _ptr(k_new),
                            _ptr(v_new), _ptr(N), _ptr(O), _ptr(ws), ws.numel(), _stream(stream)))


def dense(cfg: Config, K, V, Q, N, O, ws, n_q: int = 1, stream=None):
    _check(lib().zha_dense(ctypes.byref(cfg.c()), _ptr(K), _ptr(V), _ptr(Q), n_q, _ptr(N), _ptr(O), _ptr(ws),
                           ws.numel(), _stream(stream)))


def get_status(clear: bool = True, stream=None) -> int:
    v = ctypes.c_int32()
    _check(lib().zha_get_status(ctypes.byref(v), 1 if clear else 0, _stream(stream)))
    return v.value


def status_names(bits: int) -> list[str]:
    return [STATUS[c] for c in STATUS if c and bits & (1 << c)]


def set_wait_limit(ns: int) -> int:
    """Sets the bound (ns) of the tensor-core decode attention's waits on its other warps'
    progress; returns the previous bound (see include/zha.h, zha_set_wait_limit)."""
    prev = ctypes.c_uint64()
    _check(lib().zha_set_wait_limit(int(ns), ctypes.byref(prev)))
    return prev.value
