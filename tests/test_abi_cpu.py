"""The C-ABI library loads and exports every symbol include/zha.h declares, and
its host-side checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from hierarchical_tree_indexed_b200 import build_lib, zha

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return zha.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "zha.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 13, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in zha.h but not exported"
    assert set(names) <= set(zha.EXPORTS) | {"zha_last_error"}


def test_struct_layout_matches_header():
    # int32 x 8, int64, int32, float, float[16], int32 -> 8*4 + 8 + 4 + 4 + 64 + 4 = 116 bytes,
    # padded to the int64's alignment: 120
    assert ctypes.sizeof(zha.ZhaConfig) == 120
    assert zha.ZhaConfig.N_cap.offset == 32 and zha.ZhaConfig.p.offset == 48 and zha.ZhaConfig.vsum.offset == 112


def cfg(**kw):
    base = dict(d=128, Hq=32, Hkv=8, B=64, b=16, batch=4, N_cap=1048576 + 64)
    base.update(kw)
    return zha.Config(**base)


def test_sizes_and_levels(lib):
    assert zha.levels_cap(cfg()) == 4
    assert zha.levels_cap(cfg(batch=1, N_cap=8388608 + 256)) == 5
    assert zha.levels_cap(cfg(N_cap=4096, B=16, b=4, d=64, Hq=1, Hkv=1, batch=1, dtype="f32")) == 4
    assert zha.levels_cap(cfg(N_cap=262144, B=4, b=4, L_fixed=6)) == 6
    # summaries of every level: (16385 + 1025 + 65 + 5) nodes x (512 + 4) B x 32 slices, plus small parts
    tb = zha.tree_bytes(cfg())
    assert 16385 * 516 * 32 < tb < 17600 * 516 * 32
    assert zha.workspace_bytes(cfg()) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(R=17), 2), (dict(Hq=30), 1), (dict(Hq=64), 2), (dict(B=0), 1),
    (dict(B=512), 2), (dict(b=1), 1), (dict(b=64), 2), (dict(batch=0), 1), (dict(N_cap=0), 1),
    (dict(p=0.0), 1), (dict(p=float("nan")), 1), (dict(L_fixed=17), 1), (dict(scale=-1.0), 1),
    (dict(vsum=2), 1), (dict(vsum=1, R=2), 2),
])
def test_config_validation(lib, kw, code):
    with pytest.raises(zha.ZhaError) as e:
        zha.tree_bytes(cfg(**kw))
    assert e.value.code == code
    assert lib.zha_last_error().decode()


def test_null_pointers_and_small_workspace_are_refused_on_the_host(lib):
    c = cfg(batch=1, N_cap=4096)
    cc = ctypes.byref(c.c())
    assert lib.zha_build(cc, None, None, None, None, None, None) == 1
    assert lib.zha_extend(cc, None, None, None, None, None) == 1
    cv = ctypes.byref(cfg(batch=1, N_cap=4096, vsum=1).c())                # value summaries need V
    assert lib.zha_build(cv, 1, None, 1, 1, 1, None) == 1
    with pytest.raises(zha.ZhaError) as e:                                  # no chunked prefill with them
        zha.workspace_bytes(cfg(batch=1, N_cap=4096, vsum=1), 64)
    assert e.value.code == 2
    assert lib.zha_attend_noalloc(cv, 1, 1, 1, 1, 1, 1, 1, 1, 16, 1, None) == 2   # nor the no-alloc call
    # the no-alloc call is decode only: a chunked prefill (n_q > 1) is refused before anything runs
    assert lib.zha_attend_noalloc(cc, 1, 1, 1, 1, 64, 1, 1, 1, 16, 1, None) == 2
    assert "n_q = 1" in lib.zha_last_error().decode()
    off = ctypes.c_size_t()
    assert lib.zha_tree_level_v(cc, 1, ctypes.byref(off)) == 1             # vsum = 0: no vhat
    assert lib.zha_tree_level_v(cv, 1, ctypes.byref(off)) == 0
    assert lib.zha_append(cc, None, None, None, None, None, None, None) == 1
    need = zha.workspace_bytes(c)
    assert lib.zha_route(cc, 1, 1, 1, 1, 1, 1, 16, 256, need - 1, None) == 6
    pneed = zha.workspace_bytes(c, 64)                                      # chunked prefill of 64 queries
    assert lib.zha_route(cc, 1, 1, 64, 1, 1, 1, 16, 256, pneed - 1, None) == 6
    assert lib.zha_attend(cc, 1, 1, 1, 1, 64, 1, None, 1, 16, 1, 1, pneed, None) == 1   # prefill needs sel
    cf = cfg(batch=1, N_cap=4096, dtype="f32")
    assert lib.zha_route(ctypes.byref(cf.c()), 1, 1, 64, 1, 1, 1, 16, 256, pneed, None) == 2   # bf16 only
    assert lib.zha_attend(cc, 1, 1, 1, 1, 1, 1, 1, 1, 0, 1, 256, need, None) == 1   # sel_cap 0
    assert lib.zha_attend(cc, 1, 1, 1, 1, 1, 1, 1, 1, 1, None, 256, need, None) == 1   # O null
    assert lib.zha_decode(cc, None, None, None, None, None, None, None, None, 256, need, None) == 1
    assert lib.zha_dense(cc, 1, 1, 1, 1, 1, 1, None, need, None) == 1
    assert "ws" in lib.zha_last_error().decode()


def test_wait_limit_setter_round_trips(lib):
    prev = zha.set_wait_limit(12345)
    try:
        assert zha.set_wait_limit(prev) == 12345
    finally:
        zha.set_wait_limit(prev)
    assert prev == 2_000_000_000
