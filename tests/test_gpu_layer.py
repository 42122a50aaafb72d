"""GPU parity of the layer / stack path (through the C ABI) against the
float64 oracle on the same seeded inputs.

Tolerances (written here):
* the layer output Y (spec bound): max |gpu - oracle| / RMS(oracle)
  <= 1e-4 (fp32 workloads), <= 2e-2 (bf16 workloads);
* the pre-LayerNorm attention output O (kept in fp32 by the kernels): the
  same bound;
* the gated Z = LayerNorm(O) * U, three ways: (i) the LayerNorm * U step on
  its own, i.e. Z against the oracle's LayerNorm * U of the GPU's own O and U,
  by the max metric at the same bound; (ii) Z against the oracle's Z,
  element by element, within the first-order bound of LayerNorm's
  amplification of the upstream errors: |dZ_k| <= |gamma_k U_k| * max|dO| *
  (2 + |xhat_k|) / sigma + |LN(O)_k| * |dU_k|, doubled, plus Z's own fp16
  rounding (sigma is the row's standard deviation: a row whose O varies
  little amplifies O's error most, so a max metric normalised by the whole
  tensor's RMS would measure O's error times the largest amplification, not
  the step); (iii) RMS-normalised RMS error at the same bound;
* the layer delta Y - X: RMS-normalised RMS error at the same bound (its max
  error contains Y's own bf16 rounding, which scales with |Y|, not the delta);
* the f1 output (U|V|Q|K after SiLU), which the tensor-core path stores in
  fp16: within one fp16 ulp of the oracle's exact value plus 1e-4 of its RMS
  (the fp32 accumulation floor near zero); a stored 16-bit tensor's max/RMS
  error is bounded below by its own rounding.
"""
import math

import numpy as np
import pytest

import hstu_workloads as hw
from oracle import hstu_oracle as O
from gpu_util import TOL, decode_o, relerr, rmserr, run_stack, runner_for, ulperr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    from hstu_sequential_transducer_layer_b200 import binding as B
    build()
    B.hstu_debug_keep_z(True)      # the layer calls of this module also write Z
    yield
    B.hstu_debug_keep_z(False)


def z_checks(z, o, u, z_ref, o_ref, u_ref, gamma, beta, eps):
    """The three checks of the gated Z described in the module docstring:
    returns (step max-metric error, worst ratio of the error to its derived
    bound, RMS-normalised RMS error)."""
    g = gamma.astype(np.float64)
    b = beta.astype(np.float64)
    step = relerr(z, O.layer_norm(o, g, b, eps) * u)
    mu = o_ref.mean(axis=1, keepdims=True)
    sig = np.sqrt(o_ref.var(axis=1, keepdims=True) + eps)
    xhat = (o_ref - mu) / sig
    d_o = np.abs(o - o_ref).max(axis=1, keepdims=True)
    ln = xhat * g + b
    bound = 2.0 * (np.abs(g * u) * d_o * (2.0 + np.abs(xhat)) / sig + np.abs(ln) * np.abs(u - u_ref))
    bound += 2.0 ** -10 * np.abs(z_ref) + 1e-6 * math.sqrt(float(np.mean(z_ref ** 2)))
    ratio = float(np.max(np.abs(z - z_ref) / bound)) if z.size else 0.0
    return step, ratio, rmserr(z, z_ref)


def _check_layer(w, tol, Y, runner):
    ref, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims,
                             return_intermediates=True)
    f1, o, z = runner.intermediates(w.B, w.T, w.max_len)
    f1, z = f1.double().cpu().numpy(), z.double().cpu().numpy()
    o = decode_o(o, w.dims.n_heads, w.dims.d_v)
    X = w.X.astype(np.float64)
    hdv = w.dims.n_heads * w.dims.d_v
    lw = w.weights[0]
    z_step, z_bound, z_rms = z_checks(z, o, f1[:, :hdv], inter["Z"], inter["O"], inter["G"][:, :hdv],
                                      lw["ln_gamma"], lw["ln_beta"], w.dims.ln_eps)
    errs = dict(Y=relerr(Y, ref), O=relerr(o, inter["O"]), Z_step=z_step, Z_rms=z_rms,
                dY=rmserr(Y - X, ref - X))
    if w.dims.dtype == hw.BF16:
        errs["G_ulp"] = ulperr(f1, inter["G"])
    else:
        errs["G"] = relerr(f1, inter["G"])
    errs["Z_bound"] = z_bound
    print(w.name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= (1.0 if k in ("G_ulp", "Z_bound") else tol), (k, v, errs)
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


def _fp16_range(a) -> float:
    return float(np.max(np.abs(a))) if np.size(a) else 0.0


def test_small_magnitude_weights_below_fp16_normal_range():
    """W2 drawn from N(0, 1e-5): nearly every value lies below fp16's smallest
    normal (2^-14) and becomes an fp16 subnormal in the tensor-core operand
    (absolute spacing 2^-24).  gamma = 8192 (beta = 0, biases 0) makes the f2
    term carry the layer delta (about a third of the output), so a conversion that lost those values (a
    flush to zero) would miss the delta entirely; subnormal rounding costs
    about 0.2% of it."""
    dims = hw.LayerDims(128, 4, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("tinyW2", [300, 129, 1, 64, 200], dims, seed=70)
    lw = w.weights[0]
    rng = np.random.default_rng(71)
    lw["W2"] = hw.round_to_bf16(rng.normal(0.0, 1e-5, size=lw["W2"].shape).astype(np.float32))
    lw["b1"][:] = 0.0
    lw["b2"][:] = 0.0
    lw["ln_gamma"][:] = 8192.0
    lw["ln_beta"][:] = 0.0
    assert np.mean(np.abs(lw["W2"]) < 2.0 ** -14) > 0.99
    Y, r, _ = run_stack(w)
    ref, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, lw, dims, return_intermediates=True)
    assert _fp16_range(inter["Z"]) < 60000.0          # the case stays inside the fp16 contract
    X = w.X.astype(np.float64)
    e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
    print("small W2", e, ed, float(np.sqrt(np.mean((ref - X) ** 2))))
    assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16]


def test_residual_stream_near_fp16_limit():
    """A 3-layer stack whose fp16 residual stream grows to about 3/4 of fp16's
    largest value (65504) and stays inside it, with every weight inside
    fp16's normal range: X of scale 8192; the Q and K rows of W1 of magnitude
    2^-14 to 2^-13 with random signs (the scores, and the P the kernel stores
    in fp16, stay within a few thousand), the U rows of W1 scaled by 1/8 (so
    the gated Z stays inside fp16), W2 by 8 (each layer's delta about half the
    residual).  The bf16 output's own rounding is up to 2^-9 of |Y| here, with
    max|Y| / RMS(Y) about 4.5."""
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("bigres", [300, 129, 1, 64], dims, n_layers=3, seed=72, x_scale=8192.0)
    hdv = 2 * 64
    rng = np.random.default_rng(73)
    for lw in w.weights:
        W1 = lw["W1"].astype(np.float64)
        W1[:hdv] /= 8.0                                  # U
        shp = W1[2 * hdv:].shape                         # Q and K
        W1[2 * hdv:] = rng.choice([-1.0, 1.0], size=shp) * 2.0 ** -14 * (1.0 + rng.random(shp))
        lw["W1"] = hw.round_to_bf16(W1.astype(np.float32))
        lw["W2"] = hw.round_to_bf16((lw["W2"] * 8.0).astype(np.float32))
        assert np.abs(lw["W1"][2 * hdv:]).min() >= 2.0 ** -14
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    # every layer output and every stored intermediate of the oracle inside fp16
    xl = w.X
    peak = 0.0
    for lw in w.weights:
        y, inter = O.layer_fwd(xl, w.offsets, w.timestamps, lw, dims, return_intermediates=True)
        peak = max(peak, _fp16_range(y), _fp16_range(inter["G"]), _fp16_range(inter["Z"]))
        xl = y
    assert 40000.0 < peak < 60000.0, peak
    Y, _, _ = run_stack(w)
    X = w.X.astype(np.float64)
    e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
    print("near-limit residual", peak, e, ed)
    assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16]


@pytest.mark.parametrize("D", [64, 128])
def test_ln_fusion_on_and_off_match_oracle(D):
    """LayerNorm * U formed inside f2's operand stage (ln_fusion = 1) and by a
    separate kernel (0): both within the bound of the oracle on
    a ragged 3-layer stack (and so within twice the bound of each other: the
    fused path computes Z in packed fp16, the separate kernel in fp32)."""
    from hstu_sequential_transducer_layer_b200 import binding as B
    dims = hw.LayerDims(256, 2, D, D, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom(f"lnfuse{D}", [300, 129, 1, 64, 0, 257], dims, n_layers=3, seed=95 + D)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    X = w.X.astype(np.float64)
    out = {}
    try:
        for f in (0, 1):
            B.hstu_set_option("ln_fusion", f)
            Y, _, _ = run_stack(w)
            out[f] = Y
            e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
            print("ln_fusion", f, D, e, ed)
            assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16], (f, e, ed)
    finally:
        B.hstu_set_option("ln_fusion", 2)
    assert relerr(out[1], out[0]) <= 2 * TOL[hw.BF16]


@pytest.mark.parametrize("last", [900, 1000])
def test_gemm_pair_on_and_off_match_oracle(last):
    """The SiLU projection f1 on CTA pairs (256-row pair MMA, gemm_pair = 2,
    which forces pairs at this K = 512) and on single CTAs (0): both within
    the bound of the oracle on a ragged 2-layer stack whose f1 takes
    256-column tiles (f1 width 2048; 4,900 rows: the last 256-row tile leaves
    the second CTA of its pair without a valid row; 5,000 rows: with 8), and
    identical to each other (the same fp32 accumulation order over K for
    every output element)."""
    from hstu_sequential_transducer_layer_b200 import binding as B
    dims = hw.LayerDims(512, 4, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    lengths = [777, 1024, 513, 1, last, 1685]
    assert sum(lengths) in (4900, 5000) and dims.f1_width == 2048
    w = hw.custom(f"pair{last}", lengths, dims, n_layers=2, seed=417)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    X = w.X.astype(np.float64)
    out = {}
    try:
        for p in (0, 2):
            B.hstu_set_option("gemm_pair", p)
            Y, _, _ = run_stack(w)
            out[p] = Y
            e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
            print("gemm_pair", p, e, ed)
            assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16], (p, e, ed)
    finally:
        B.hstu_set_option("gemm_pair", 1)
    assert np.array_equal(out[0], out[2])


def test_gemm_pair_default_at_d1024_is_bitwise_single_cta():
    """At d_model = 1024 the default (gemm_pair = 1) runs f1 on CTA pairs:
    within the oracle's bound on a ragged layer of 2,700 rows (f1 width 4096,
    256-column tiles) and bitwise equal to single CTAs (gemm_pair = 0)."""
    from hstu_sequential_transducer_layer_b200 import binding as B
    dims = hw.LayerDims(1024, 8, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    lengths = [700, 129, 1, 1024, 846]
    assert sum(lengths) == 2700 and dims.f1_width == 4096
    w = hw.custom("pair1024", lengths, dims, n_layers=1, seed=418)
    ref = O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims)
    X = w.X.astype(np.float64)
    out = {}
    try:
        for p in (0, 1):
            B.hstu_set_option("gemm_pair", p)
            Y, _, _ = run_stack(w)
            out[p] = Y
            e, ed = relerr(Y, ref), rmserr(Y - X, ref - X)
            print("gemm_pair", p, e, ed)
            assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16], (p, e, ed)
    finally:
        B.hstu_set_option("gemm_pair", 1)
    assert np.array_equal(out[0], out[1])
