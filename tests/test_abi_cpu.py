"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/hstu.h declares, sizes workspaces, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re

import pytest

import hstu_sequential_transducer_layer_b200 as H
from hstu_sequential_transducer_layer_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _declared():
    src = open(os.path.join(ROOT, "include", "hstu.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 12
    assert sorted(B.EXPORTED) == names
    L = B.lib()
    for n in names:
        assert hasattr(L, n), n
    assert H.hstu_version() == 1


def _desc(dtype="bf16", d=256, h=4, dqk=64, dv=64):
    return B.make_desc(d, h, dqk, dv, 128, 128, 4, 2, 1e-6, dtype)


def test_workspace_size_grows_with_work():
    d = _desc()
    a = B.hstu_workspace_size(d, 1, 4, 1000, 512)
    b = B.hstu_workspace_size(d, 1, 4, 2000, 512)
    c = B.hstu_workspace_size(d, 3, 4, 2000, 1024, 4096, 1024, 256)
    assert 0 < a < b < c
    assert a % 256 == 0


def test_workspace_size_rejects_bad_shapes():
    L = B.lib()
    bad = [_desc(dqk=96, dv=96), _desc(d=200), _desc(dqk=64, dv=128)]
    for d in bad:
        assert L.hstu_workspace_size(ctypes.byref(d), 1, 4, 100, 64, 0, 0, 0) == 0
    d = _desc()
    assert L.hstu_workspace_size(ctypes.byref(d), 1, 4, 1000, 64, 0, 0, 0) == 0  # T > B*max_len
    assert L.hstu_workspace_size(ctypes.byref(d), 0, 4, 100, 64, 0, 0, 0) == 0
    assert L.hstu_workspace_size(ctypes.byref(d), 1, 4, 100, 64, 10, 5, 0) == 0  # no microbatch
    f = _desc("fp32", d=64, h=2, dqk=32, dv=32)
    assert L.hstu_workspace_size(ctypes.byref(f), 1, 4, 100, 64, 0, 0, 0) > 0
    f = _desc("fp32", d=64, h=2, dqk=256, dv=32)
    assert L.hstu_workspace_size(ctypes.byref(f), 1, 4, 100, 64, 0, 0, 0) == 0


def test_bad_arguments_return_before_launch():
    L = B.lib()
    d = _desc()
    w = B.LayerWeights(*([0x1000] * 8))
    n0 = H.hstu_launch_count()
    # null offsets / workspace
    r = L.hstu_layer_fwd(ctypes.byref(d), 2, 10, 8, None, 0x1000, ctypes.byref(w), 0x1000,
                         0x2000, 0x10000, 1 << 20, None)
    assert r == 1
    # misaligned X
    r = L.hstu_layer_fwd(ctypes.byref(d), 2, 10, 8, 0x1000, 0x1008, ctypes.byref(w), 0x1000,
                         0x2000, 0x10000, 1 << 20, None)
    assert r == 1
    # X aliases out
    r = L.hstu_layer_fwd(ctypes.byref(d), 2, 10, 8, 0x1000, 0x2000, ctypes.byref(w), 0x1000,
                         0x2000, 0x10000, 1 << 20, None)
    assert r == 1
    # workspace too small
    r = L.hstu_layer_fwd(ctypes.byref(d), 2, 10, 8, 0x1000, 0x3000, ctypes.byref(w), 0x1000,
                         0x2000, 0x10000, 64, None)
    assert r == 3
    # unsupported head width
    d2 = _desc(dqk=32, dv=32)
    r = L.hstu_layer_fwd(ctypes.byref(d2), 2, 10, 8, 0x1000, 0x3000, ctypes.byref(w), 0x1000,
                         0x2000, 0x10000, 1 << 20, None)
    assert r == 2
    # null weight pointer
    w0 = B.LayerWeights(*([0x1000] * 7 + [0]))
    r = L.hstu_layer_fwd(ctypes.byref(d), 2, 10, 8, 0x1000, 0x3000, ctypes.byref(w0), 0x1000,
                         0x2000, 0x10000, 1 << 20, None)
    assert r == 1
    # M-FALCON: microbatch 0, more candidates than B * max_cands
    r = L.hstu_mfalcon_rank(ctypes.byref(d), 1, ctypes.byref(w), 2, 10, 8, 0x1000, 0x3000, 0x1000,
                            5, 4, 0x1000, 0x4000, None, 0, 0x5000, 0x6000, 0x10000, 1 << 30, None)
    assert r == 1
    r = L.hstu_mfalcon_rank(ctypes.byref(d), 1, ctypes.byref(w), 2, 10, 8, 0x1000, 0x3000, 0x1000,
                            50, 4, 0x1000, 0x4000, None, 2, 0x5000, 0x6000, 0x10000, 1 << 30, None)
    assert r == 1
    assert H.hstu_launch_count() == n0


def test_debug_offsets_and_strings():
    d = _desc()
    f1, o, z = H.hstu_debug_offsets(d, 4, 1000, 512)
    assert 0 < f1 < o < z and f1 % 256 == 0
    assert H.hstu_status_string(5).startswith("bad offsets")
    assert H.hstu_kernel_name(2) == "gemm_f1_tc"
    assert H.hstu_kernel_name(999) == "unknown"


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(B.HstuError):
        B.lib()


def test_host_keep_count_matches_oracle():
    """The library's host keep count (used to size the kept batch) equals the
    oracle's for every supported raw length, and refuses the rest."""
    from oracle import stochastic_length as SL
    got = [B.hstu_sl_keep_count(n) for n in range(0, 32768)]
    assert got == [SL.keep_count(n) for n in range(0, 32768)]
    assert B.hstu_sl_keep_count(-1) == -1 and B.hstu_sl_keep_count(32768) == -1
