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


def test_new_entry_points_reject_bad_arguments_before_launch():
    """Stochastic Length, retrieval, the comparator layer and the weight
    conversion check their arguments on the host and launch nothing when they
    are wrong (no GPU is needed to see it)."""
    L = B.lib()
    n0 = H.hstu_launch_count()
    ws, big = 0x100000, 1 << 30
    # Stochastic Length + embedding: d % 8, max_raw_len bound, workspace, nulls, alignment
    sl = lambda **k: L.hstu_sl_embed(
        k.get("B", 2), k.get("R", 10), k.get("maxlen", 8), 0x1000, k.get("ids", 0x2000), 0x3000,
        7, k.get("ctab", 0x4000), 100, 0x5000, 8, k.get("d", 64), 0x6000, 0x7000, 0x8000,
        k.get("ws", ws), k.get("wsb", 256), None)
    assert sl(d=12) == 1
    assert sl(maxlen=40000) == 2
    assert sl(ws=ws + 8) == 3 and sl(wsb=128) == 3
    assert sl(ids=None) == 1
    assert sl(ctab=0x4008) == 1
    # retrieval: sizes
    assert L.hstu_retrieval_workspace_size(4, 100, 64, 101, 0) == 0      # K > items
    assert L.hstu_retrieval_workspace_size(4, 5000, 96, 10, 0) == 0      # d % 64
    assert L.hstu_retrieval_workspace_size(70000, 5000, 64, 10, 0) == 0  # too many users
    assert L.hstu_retrieval_workspace_size(4, 5000, 64, 2000, 0) == 0    # K > 1024
    assert L.hstu_retrieval_workspace_size(4, 5000, 64, 10, 0) > 0
    # the filtering path's buffers appear only for large catalogs
    small = L.hstu_retrieval_workspace_size(128, 65535, 64, 100, 0)
    large = L.hstu_retrieval_workspace_size(128, 65536, 64, 100, 0)
    assert large > small + 128 * 16384 * 8
    need = L.hstu_retrieval_workspace_size(4, 5000, 64, 10, 0)
    ret = lambda **k: L.hstu_retrieval_topk(4, 5000, 64, k.get("H", 0x1000), None, 0, 0x2000,
                                            k.get("K", 10), 0x3000, 0x4000, k.get("ws", ws),
                                            k.get("wsb", need), None)
    assert ret(K=0) == 1 and ret(K=5001) == 1
    assert ret(wsb=need - 1) == 3 and ret(ws=ws + 16) == 3
    assert ret(H=0x1008) == 1 and ret(H=None) == 1
    taken = ctypes.c_int32(0)
    assert L.hstu_retrieval_fallback_taken(None, 256, ctypes.byref(taken), None) == 1
    # comparator layer: shapes it does not run
    assert L.hstu_transformer_workspace_size(300, 4, 1024, 2, 100) == 0   # d % 256
    assert L.hstu_transformer_workspace_size(256, 8, 1024, 2, 100) == 0   # head dim 32
    assert L.hstu_transformer_workspace_size(256, 4, 100, 2, 100) == 0    # d_ff % 256
    assert L.hstu_transformer_workspace_size(512, 8, 2048, 2, 100) > 0
    tw = B.TransformerWeights(*([0x1000] * 10))
    tneed = L.hstu_transformer_workspace_size(512, 8, 2048, 2, 100)
    tf = lambda **k: L.hstu_transformer_layer_fwd(
        k.get("d", 512), 8, 2048, 1e-6, ctypes.byref(k.get("w", tw)), 2, 100, 64, 0x1000,
        k.get("X", 0x2000), 0x3000, ws, k.get("wsb", tneed), None)
    assert tf(d=300) == 1
    assert tf(wsb=tneed - 1) == 3
    assert tf(w=B.TransformerWeights(*([0x1000] * 9 + [0]))) == 1
    assert tf(X=0x2004) == 1
    # bf16 -> fp16: length and alignment
    assert L.hstu_bf16_to_f16(0x1000, 0x2000, 7, None) == 1
    assert L.hstu_bf16_to_f16(0x1002, 0x2000, 8, None) == 1
    assert L.hstu_bf16_to_f16(0x1000, 0x2000, 0, None) == 0
    assert H.hstu_launch_count() == n0


def test_option_and_test_hook_arguments_checked():
    """Process-wide options and test hooks reject what they do not know
    (host only, nothing launched)."""
    L = B.lib()
    assert L.hstu_set_option(b"ln_fusion", 3) == 1
    assert L.hstu_set_option(b"ln_fusion", -1) == 1
    assert L.hstu_set_option(b"no_such_option", 0) == 1
    assert L.hstu_set_option(None, 0) == 1
    assert L.hstu_set_option(b"ln_fusion", 1) == 0
    assert L.hstu_set_option(b"ln_fusion", 0) == 0
    assert L.hstu_set_option(b"ln_fusion", 2) == 0
    assert L.hstu_set_option(b"gemm_pair", 3) == 1
    assert L.hstu_set_option(b"gemm_pair", -1) == 1
    assert L.hstu_set_option(b"gemm_pair", 0) == 0
    assert L.hstu_set_option(b"gemm_pair", 2) == 0
    assert L.hstu_set_option(b"gemm_pair", 1) == 0
    assert L.hstu_debug_keep_z(3) == 1
    assert L.hstu_debug_wait_test(1000, 5) == 1
    assert L.hstu_debug_wait_test(0, 0) == 0
    assert L.hstu_trace_only(-2) == 1
    assert L.hstu_trace_only(100000) == 1
    assert L.hstu_trace_only(2) == 0
    assert L.hstu_trace_only(-1) == 0
    assert L.hstu_last_error() is not None


def test_bwd_workspace_and_argument_errors():
    L = B.lib()
    d = _desc()
    a = B.hstu_bwd_workspace_size(d, 1, 4, 1000, 512)
    b = B.hstu_bwd_workspace_size(d, 2, 4, 1000, 512)
    assert 0 < a < b and a % 256 == 0
    f = _desc("fp32", d=64, h=2, dqk=32, dv=32)
    assert L.hstu_bwd_workspace_size(ctypes.byref(f), 1, 4, 100, 64) == 0   # bf16 only
    g = B.LayerGrads(*([0x1000] * 8))
    w = B.LayerWeights(*([0x1000] * 8))
    code = L.hstu_layer_bwd(ctypes.byref(f), ctypes.byref(w), 4, 100, 64, 0x1000, 0x1000, 0x1000,
                            0x1000, 0x1000, ctypes.byref(g), 0x1000, 1 << 20, None)
    assert code == 2  # HSTU_ERR_UNSUPPORTED, nothing launched
    code = L.hstu_layer_bwd(ctypes.byref(d), ctypes.byref(w), 4, 100, 64, 0x1000, 0x1000, 0x1000,
                            0x1000, 0x1000, ctypes.byref(g), 0x1000, 1024, None)
    assert code == 3  # workspace too small
    bad = B.LayerGrads(*([0x1000] * 7 + [0]))
    code = L.hstu_layer_bwd(ctypes.byref(d), ctypes.byref(w), 4, 100, 64, 0x1000, 0x1000, 0x1000,
                            0x1000, 0x1000, ctypes.byref(bad), 0x1000, 1 << 40, None)
    assert code == 1  # a null gradient pointer
