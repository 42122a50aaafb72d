"""GPU parity of the backward pass (hstu_layer_bwd / hstu_stack_bwd, through
the C ABI) against the float64 backward oracle (oracle.hstu_backward, itself
pinned by finite differences and torch autograd) on the same seeded inputs.

Tolerance (written here): every gradient -- dX and each parameter's --
within max |gpu - oracle| / RMS(oracle) <= 2e-2, the bf16 bound of the
forward parity tests, and within RMS-normalised RMS error <= 2e-2.  Two
exceptions, both in the stack test and both from one ill-conditioned row:
the dX row of a user of one token is held to the RMS bound only, and the
bottom layer's dW1 (which sums that row's dP times its input) to a max
metric of 3e-2.  That row's gradient is ill-conditioned with respect to the
fp16 rounding of the layer's f1 output: an emulation of the kernels'
rounding points in float64 (tests/bwd_rounding_emulation.py) puts that
row's dX error at 2.3e-2 and every
other row's at <= 2.9e-3 (RMS 4.9e-4), and the bottom layer's dW1 error at
1.99e-2, of which 1.45e-2 comes from the f1-output rounding alone; the
kernels measure 1.99e-2 to 2.01e-2, depending on how the compiler contracts
the elementwise arithmetic.  So the max metric there measures the
conditioning, not the kernels; 3e-2 is 1.5 times the emulated value.  dY is rounded to bf16 before both sides see
it (the boundary takes bf16), the weights are the workload's bf16 values.
"""
import numpy as np
import pytest

import hstu_workloads as hw
from gpu_util import TOL, relerr, rmserr, runner_for
from oracle import hstu_backward as BW

pytestmark = pytest.mark.gpu

GRAD_KEYS = ("dW1", "db1", "dW2", "db2", "dln_gamma", "dln_beta", "drab_pos", "drab_time")


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _run_bwd(w, dY, n_layers=None):
    import torch
    r = runner_for(w)
    off = r.to_device(w.offsets, "i64")
    X = r.to_device(w.X, "act")
    ts = r.to_device(w.timestamps, "i64")
    dYd = r.to_device(dY, "act")
    dX, grads = r.stack_bwd(off, X, ts, dYd, w.max_len, n_layers=n_layers)
    torch.cuda.synchronize()
    assert r.bwd_status() == 0
    return (dX.double().cpu().numpy(),
            [{k: g[k].double().cpu().numpy() for k in GRAD_KEYS} for g in grads])


def _check(name, got_dX, got, ref_dX, ref, dx_rows=None, loose=None):
    """dx_rows: the dX rows held to the max metric (default all); loose:
    max-metric bounds other than the bf16 one, by key."""
    rows = slice(None) if dx_rows is None else dx_rows
    rms_ref = float(np.sqrt(np.mean(ref_dX ** 2)))
    errs = {"dX": float(np.abs(got_dX[rows] - ref_dX[rows]).max()) / rms_ref,
            "dX_rms": rmserr(got_dX, ref_dX)}
    for layer, (g, rg) in enumerate(zip(got, ref)):
        for k in GRAD_KEYS:
            errs[f"{k}[{layer}]"] = relerr(g[k], rg[k])
            errs[f"{k}[{layer}]_rms"] = rmserr(g[k], rg[k])
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= (loose or {}).get(k, TOL[hw.BF16]), (k, v)


@pytest.mark.parametrize("D", [64, 128])
def test_layer_bwd_ragged_matches_oracle(D):
    dims = hw.LayerDims(128, 2, D, D, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom(f"bwd{D}", [1, 127, 128, 129, 300, 0, 5, 257], dims, seed=80 + D)
    dY = hw.round_to_bf16(np.random.default_rng(81).standard_normal(w.X.shape).astype(np.float32))
    dX, grads = _run_bwd(w, dY)
    ref = BW.layer_bwd(w.X, w.offsets, w.timestamps, w.weights[0], dims, dY)
    ref_dX = ref.pop("dX")
    _check(f"layer D={D}", dX, grads, ref_dX, [ref])


def test_stack_bwd_two_layers_matches_oracle():
    dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom("bwdstack", [300, 129, 1, 64, 0, 200], dims, n_layers=2, seed=82)
    dY = hw.round_to_bf16(np.random.default_rng(83).standard_normal(w.X.shape).astype(np.float32))
    dX, grads = _run_bwd(w, dY)
    ref_dX, ref = BW.stack_bwd(w.X, w.offsets, w.timestamps, w.weights, dims, dY)
    lens = np.diff(w.offsets)
    multi = np.repeat(lens >= 2, lens)          # rows of users with two or more tokens
    _check("stack of 2", dX, grads, ref_dX, ref, dx_rows=multi, loose={"dW1[0]": 3e-2})


def test_bwd_deterministic():
    """Two calls on the same inputs give bit-identical gradients, the bias
    tables' included (their sums are fixed-point integers, so the order of the
    kernel's additions does not matter)."""
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("bwddet", [200, 3, 130], dims, seed=84)
    dY = hw.round_to_bf16(np.random.default_rng(85).standard_normal(w.X.shape).astype(np.float32))
    a_dX, a = _run_bwd(w, dY)
    b_dX, b = _run_bwd(w, dY)
    assert np.array_equal(a_dX, b_dX)
    for k in GRAD_KEYS:
        assert np.array_equal(a[0][k], b[0][k]), k


def test_bwd_no_rows_gives_zero_gradients():
    import torch
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("bwdempty", [0, 0], dims, seed=86)
    r = runner_for(w)
    off = r.to_device(w.offsets, "i64")
    X = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    ts = torch.zeros(0, dtype=torch.int64, device="cuda")
    dX, grads = r.stack_bwd(off, X, ts, X, 1)
    torch.cuda.synchronize()
    assert r.bwd_status() == 0 and dX.shape == (0, 128)
    for k in GRAD_KEYS:
        assert float(grads[0][k].abs().max()) == 0.0, k


def test_bwd_pairs_bitwise():
    """The backward call's forward keeps f1's pre-activation next to G; with
    f1 forced onto CTA pairs (gemm_pair = 2) on a case whose f1 takes
    256-column tiles (f1 width 2048, 5,000 rows), every gradient and dX is
    bitwise the single-CTA run's."""
    from hstu_sequential_transducer_layer_b200 import binding as B
    dims = hw.LayerDims(512, 4, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom("bwdpair", [777, 1024, 513, 1, 1000, 1685], dims, n_layers=2, seed=87)
    dY = hw.round_to_bf16(np.random.default_rng(88).standard_normal(w.X.shape).astype(np.float32))
    out = {}
    try:
        for p in (0, 2):
            B.hstu_set_option("gemm_pair", p)
            out[p] = _run_bwd(w, dY)
    finally:
        B.hstu_set_option("gemm_pair", 1)
    assert np.array_equal(out[0][0], out[2][0])
    for layer in range(2):
        for k in GRAD_KEYS:
            assert np.array_equal(out[0][1][layer][k], out[2][1][layer][k]), (layer, k)
