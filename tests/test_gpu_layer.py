"""GPU parity of the layer / stack path (through the C ABI) against the
float64 oracle on the same seeded inputs.

Tolerances (written here):
* the layer output Y (spec bound): max |gpu - oracle| / RMS(oracle)
  <= 1e-4 (fp32 workloads), <= 2e-2 (bf16 workloads);
* the pre-LayerNorm attention output O (kept in fp32 by the kernels): the
  same bound;
* the gated Z = LayerNorm(O) * U (an intermediate whose max error is
  LayerNorm-amplified where a row's variance is small): RMS-normalised RMS
  error at the same bound;
* the layer delta Y - X: RMS-normalised RMS error at the same bound (its max
  error contains Y's own bf16 rounding, which scales with |Y|, not the delta);
* the f1 output (U|V|Q|K after SiLU), which the tensor-core path stores in
  fp16: within one fp16 ulp of the oracle's exact value plus 1e-4 of its RMS
  (the fp32 accumulation floor near zero); a stored 16-bit tensor's max/RMS
  error is bounded below by its own rounding.
"""
import numpy as np
import pytest

import hstu_workloads as hw
from oracle import hstu_oracle as O
from gpu_util import TOL, relerr, rmserr, run_stack, runner_for, ulperr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _check_layer(w, tol, Y, runner):
    ref, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims,
                             return_intermediates=True)
    f1, o, z = (t.double().cpu().numpy() for t in runner.intermediates(w.B, w.T, w.max_len))
    X = w.X.astype(np.float64)
    errs = dict(Y=relerr(Y, ref), O=relerr(o, inter["O"]), Z_rms=rmserr(z, inter["Z"]),
                dY=rmserr(Y - X, ref - X))
    if w.dims.dtype == hw.BF16:
        errs["G_ulp"] = ulperr(f1, inter["G"])
    else:
        errs["G"] = relerr(f1, inter["G"])
    print(w.name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= (1.0 if k == "G_ulp" else tol), (k, v, errs)
    return errs


def test_tiny_fp32_matches_oracle():
    w = hw.tiny_fp32(0)
    Y, r, _ = run_stack(w)
    _check_layer(w, TOL[hw.FP32], Y, r)


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_ragged_tiles_match_oracle(D):
    dims = hw.LayerDims(128, 2, D, D, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom(f"ragged{D}", [1, 127, 128, 129, 300, 0, 5, 257], dims, seed=40 + D)
    Y, r, _ = run_stack(w)
    _check_layer(w, TOL[hw.BF16], Y, r)


def test_bf16_epochs_and_unsorted_timestamps():
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("epochs", [200, 3, 150], dims, seed=44,
                  ts_base=[1_700_000_000, 5, 1 << 40])
    w.timestamps[10] += 100000        # out of order inside user 0
    w.timestamps[205] -= 3            # and inside user 2
    Y, r, _ = run_stack(w)
    _check_layer(w, TOL[hw.BF16], Y, r)


def test_single_layer_workload_full():
    w = hw.single_layer(0)
    Y, r, _ = run_stack(w)
    _check_layer(w, TOL[hw.BF16], Y, r)


def test_fp32_stack_three_layers():
    dims = hw.LayerDims(64, 2, 32, 16, 32, 32, 2, 0, 1e-6, hw.FP32)
    w = hw.custom("f32stack", [9, 40, 1, 77], dims, n_layers=3, seed=45, init="normal")
    Y, _, _ = run_stack(w)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    assert relerr(Y, ref) <= TOL[hw.FP32]


def test_bf16_stack_three_layers():
    dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom("bf16stack", [300, 129, 1, 64], dims, n_layers=3, seed=46)
    Y, _, _ = run_stack(w)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    X = w.X.astype(np.float64)
    e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
    print("bf16 stack", e, ed)
    assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16]


def test_weights_converted_per_call_or_once_agree():
    """The fp16 weight copies made once at load time (W1_f16 / W2_f16) and
    the per-call conversion into the workspace give the same bits, and both
    match the oracle."""
    dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom("f16w", [300, 129, 1, 64], dims, n_layers=3, seed=47)
    Y1, _, _ = run_stack(w, runner=runner_for(w, f16_weights=True))
    Y0, _, _ = run_stack(w, runner=runner_for(w, f16_weights=False))
    np.testing.assert_array_equal(Y1, Y0)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    assert relerr(Y1, ref) <= TOL[hw.BF16]


def _sampled_rows_check(w, Y, users, rows_per_user=6, seed=0):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for b in users:
        s, e = int(w.offsets[b]), int(w.offsets[b + 1])
        n = e - s
        rows = np.unique(np.r_[[0, min(1, n - 1), min(127, n - 1), min(128, n - 1), n // 2, n - 1],
                               rng.integers(0, n, rows_per_user)])
        ref, _ = O.layer_rows(w.X[s:e], w.timestamps[s:e], w.weights[0], w.dims, rows)
        err = relerr(Y[s + rows], ref)
        worst = max(worst, err)
    return worst


def test_long_history_sampled_rows():
    """Full-size 8192-cap workload in the bench's launch configuration; the
    oracle computes sampled rows of the shortest, the longest and one middle user."""
    w = hw.long_history(0)
    Y, _, _ = run_stack(w)
    lens = w.lengths
    users = [int(np.argmin(lens)), int(np.argmax(lens)), int(np.argsort(lens)[len(lens) // 2])]
    err = _sampled_rows_check(w, Y, users)
    print("long_history sampled", err)
    assert err <= TOL[hw.BF16]


def test_full_stack_sampled_users():
    """Full 8-layer, d=1024 workload on the GPU; the oracle runs whole users
    (all their rows through all 8 layers) for three users incl. the longest."""
    w = hw.full_stack(0)
    Y, _, _ = run_stack(w)
    lens = w.lengths
    users = [int(np.argmax(lens)), int(np.argmin(lens)), int(np.argsort(lens)[len(lens) // 2])]
    for b in users:
        s, e = int(w.offsets[b]), int(w.offsets[b + 1])
        ref = O.stack_user(w.X[s:e], w.timestamps[s:e], w.weights, w.dims)
        X = w.X[s:e].astype(np.float64)
        err, ed = relerr(Y[s:e], ref), rmserr(Y[s:e] - X, ref - X)
        print("full_stack user", b, lens[b], err, ed)
        assert err <= TOL[hw.BF16] and ed <= TOL[hw.BF16]


def test_causality_bitwise():
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("causal", [260, 100], dims, seed=47)
    Y0, r, _ = run_stack(w)
    cut = 131
    w.X[cut + 1:260] = hw.round_to_bf16(w.X[cut + 1:260] + 2.0)
    w.timestamps[cut + 1:260] += 7777
    Y1, _, _ = run_stack(w, runner=r)
    assert np.array_equal(Y0[:cut + 1], Y1[:cut + 1])
    assert np.array_equal(Y0[260:], Y1[260:])
    assert not np.array_equal(Y0[cut + 1:260], Y1[cut + 1:260])


def test_deterministic_repeat():
    w = hw.single_layer(1)
    Y0, r, _ = run_stack(w)
    Y1, _, _ = run_stack(w, runner=r)
    assert np.array_equal(Y0, Y1)


def test_empty_and_degenerate_batches():
    import torch
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("empty", [0, 0, 0], dims, seed=48)
    r = runner_for(w)
    off = r.to_device(w.offsets, "i64")
    X = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    ts = torch.zeros(0, dtype=torch.int64, device="cuda")
    out = r.stack(off, X, ts, 1)
    assert out.shape == (0, 128) and r.status() == 0
    w1 = hw.custom("ones", [1, 1, 1, 1], dims, seed=49)
    Y, r1, _ = run_stack(w1)
    _check_layer(w1, TOL[hw.BF16], Y, r1)


def test_device_status_bad_offsets_and_timestamps():
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("bad", [10, 20], dims, seed=50)
    r = runner_for(w)
    X = r.to_device(w.X, "act")
    ts = r.to_device(w.timestamps, "i64")
    bad = r.to_device(np.array([0, 25, 30]), "i64")          # user 1 longer than max_len 20
    r.stack(bad, X, ts, 20)
    assert r.status() == 5
    bad = r.to_device(np.array([0, 12, 29]), "i64")          # total != T
    r.stack(bad, X, ts, 64)
    assert r.status() == 5
    bad = r.to_device(np.array([0, 22, 10]), "i64")          # decreasing
    r.stack(bad, X, ts, 64)
    assert r.status() == 5
    t2 = w.timestamps.copy()
    t2[15] += 1 << 31                                         # span of 2^31 s inside user 1
    r.stack(r.to_device(w.offsets, "i64"), X, r.to_device(t2, "i64"), 64)
    assert r.status() == 7
    r.stack(r.to_device(w.offsets, "i64"), X, ts, 64)         # and a good call afterwards
    assert r.status() == 0
