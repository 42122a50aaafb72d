"""GPU parity of the softmax-Transformer comparator layer
(hstu_transformer_layer_fwd, through the C ABI) against the oracle
(oracle.transformer) on the same seeded inputs.

Tolerance (the bf16 bound of the HSTU layer, written here): the output Y
within max |gpu - oracle| / RMS(oracle) <= 2e-2, and the layer delta Y - X
within RMS-normalised RMS error <= 2e-2 (its max error contains Y's own bf16
rounding).  The GPU keeps LayerNorm outputs, Q/K/V, P (the un-normalised
softmax weights, <= 2^8), the attention output, the residual stream and the
feed-forward hidden layer in fp16, and accumulates in fp32.
"""
import numpy as np
import pytest

import hstu_workloads as hw
from oracle import transformer as TR
from gpu_util import relerr, rmserr

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _run(X, offsets, d, h, ff, w, max_len=None):
    import torch
    from hstu_sequential_transducer_layer_b200 import TransformerRunner
    r = TransformerRunner(d, h, ff, w)
    Xd = torch.from_numpy(np.ascontiguousarray(X, np.float32)).cuda().to(torch.bfloat16)
    off = torch.from_numpy(np.asarray(offsets, np.int64)).cuda()
    ml = int(max_len if max_len is not None else max(1, np.diff(offsets).max(initial=1)))
    Y = r.layer(off, Xd, ml)
    torch.cuda.synchronize()
    return r.status(), Y.double().cpu().numpy()


def _check(lengths, d, h, ff, seed):
    rng = np.random.default_rng(seed)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    X = hw.round_to_bf16(rng.standard_normal((int(offsets[-1]), d)).astype(np.float32))
    w = hw.transformer_weights(seed, d, ff)
    st, Y = _run(X, offsets, d, h, ff, w)
    assert st == 0
    ref = TR.layer_fwd(X, offsets, w, h, 1e-6)
    X64 = X.astype(np.float64)
    e, ed = relerr(Y, ref), rmserr(Y - X64, ref - X64)
    print("transformer", lengths[:4], d, h, e, ed)
    assert e <= TOL and ed <= TOL, (e, ed)


def test_ragged_head_dim_64():
    _check([1, 127, 128, 129, 300, 0, 5, 257], 256, 4, 1024, 60)


def test_ragged_head_dim_128():
    _check([200, 3, 150, 1, 384], 256, 2, 512, 61)


def test_d512_eight_heads_multi_tile():
    _check([700, 513, 64], 512, 8, 2048, 62)


def test_long_history_sampled_rows():
    """The comparison workload at full size (16 users of 2,048-8,192 tokens,
    d = 512, 8 heads, d_ff = 2048) on the GPU; the oracle computes sampled
    rows of the shortest, the longest and a middle user."""
    wl = hw.long_history(0)
    d, h, ff = 512, 8, 2048
    w = hw.transformer_weights(0, d, ff)
    st, Y = _run(wl.X, wl.offsets, d, h, ff, w, wl.max_len)
    assert st == 0
    lens = wl.lengths
    rng = np.random.default_rng(3)
    worst = 0.0
    for b in [int(np.argmin(lens)), int(np.argmax(lens)), int(np.argsort(lens)[len(lens) // 2])]:
        s, n = int(wl.offsets[b]), int(lens[b])
        rows = np.unique(np.r_[[0, 1, 127, 128, n // 2, n - 1], rng.integers(0, n, 4)])
        ref = TR.user_rows(wl.X[s:s + n], w, h, 1e-6, rows)
        worst = max(worst, relerr(Y[s + rows], ref))
    print("transformer long_history sampled", worst)
    assert worst <= TOL


def test_bad_offsets_set_status():
    import torch
    from hstu_sequential_transducer_layer_b200 import TransformerRunner
    d, h, ff = 256, 4, 512
    r = TransformerRunner(d, h, ff, hw.transformer_weights(1, d, ff))
    X = torch.zeros((50, d), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 30, 20, 50], dtype=torch.int64, device="cuda")
    r.layer(off, X, 64)
    assert r.status() == 5


def test_pairs_bitwise():
    """The comparator layer with its QKV (plain bias) and FFN (SiLU)
    projections forced onto CTA pairs (gemm_pair = 2; at d = 512 the default
    keeps single CTAs): bitwise the single-CTA result, on 7,000 ragged rows
    (both projections take 256-column tiles)."""
    from hstu_sequential_transducer_layer_b200 import binding as B
    lengths = [1500, 1, 2048, 700, 2751]
    rng = np.random.default_rng(64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    d, h, ff = 512, 8, 2048
    X = hw.round_to_bf16(rng.standard_normal((int(offsets[-1]), d)).astype(np.float32))
    w = hw.transformer_weights(64, d, ff)
    out = {}
    try:
        for p in (0, 2):
            B.hstu_set_option("gemm_pair", p)
            st, out[p] = _run(X, offsets, d, h, ff, w)
            assert st == 0
    finally:
        B.hstu_set_option("gemm_pair", 1)
    assert np.array_equal(out[0], out[2])
