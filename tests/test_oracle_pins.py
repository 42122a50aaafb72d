"""Pins of the float64 oracle against things other than itself.

* hand-derived bucket values (tests/golden/log_buckets.txt) and closed forms;
* pure-Python brute force (explicit i, j, k loops) on tiny inputs;
* a padded-and-masked dense batch vs the jagged result;
* invariants: causality, 1/n linearity, M-FALCON candidate independence,
  microbatch independence, and M-FALCON == "append one candidate, rerun";
* special cases with closed forms (n=1, V=0, Q=K=0, LayerNorm vs torch);
* planted mistakes (in a patched copy of the oracle, on the CPU) that the
  pins above must catch.
"""
import copy
import math
import os

import numpy as np
import pytest

import hstu_workloads as hw
from oracle import hstu_oracle as O
from oracle import bruteforce as BF

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "log_buckets.txt")


def _small_dims(**kw):
    base = dict(d_model=32, n_heads=2, d_qk=16, d_v=8, n_pos_buckets=32, n_time_buckets=32,
                pos_sub_bits=2, time_sub_bits=0, ln_eps=1e-6, dtype=hw.FP32)
    base.update(kw)
    return hw.LayerDims(**base)


def _relerr(a, b):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    rms = math.sqrt(float(np.mean(b * b))) or 1.0
    return float(np.max(np.abs(a - b))) / rms


# ---------------------------------------------------------------- buckets
def _golden_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            n, s, x, b = (int(v) for v in line.split())
            rows.append((n, s, x, b))
    return rows


def test_bucket_golden_values():
    rows = _golden_rows()
    assert len(rows) > 40
    for n, s, x, b in rows:
        assert int(O.log_bucket(np.array([x]), n, s)[0]) == b, (n, s, x)
        assert BF.bucket_scalar(x, n, s) == b, (n, s, x)


def test_bucket_closed_forms():
    x = np.arange(0, 5000, dtype=np.int64)
    # S = 0: the bucket is the bit length of x
    got = O.log_bucket(x, 10 ** 6, 0)
    assert np.array_equal(got, np.array([int(v).bit_length() for v in x]))
    # 2^S above every x: identity
    assert np.array_equal(O.log_bucket(x, 10 ** 6, 13), x)
    # powers of two above 2^S land on (k - S + 1) * 2^S
    for S in range(0, 6):
        for k in range(S, 40):
            assert int(O.log_bucket(np.array([1 << k]), 10 ** 9, S)[0]) == (k - S + 1) << S
    # monotone, steps of at most one, no gaps
    for S in range(0, 6):
        b = O.log_bucket(np.arange(0, 1 << 16), 10 ** 9, S)
        db = np.diff(b)
        assert db.min() >= 0 and db.max() <= 1


def test_workload_sub_bits_are_largest_fitting():
    caps = {"tiny_fp32": (64, 32), "single_layer": (1024, 128), "long_history": (8192, 128),
            "mfalcon": (4096, 128), "full_stack": (hw.stochastic_length_keep(4096), 128)}
    for name, (cap, nb) in caps.items():
        S = hw.POS_SUB_BITS[name]
        assert O.log_bucket(np.array([cap - 1]), 10 ** 9, S)[0] <= nb - 1
        assert O.log_bucket(np.array([cap - 1]), 10 ** 9, S + 1)[0] > nb - 1
    for nb, S in hw.TIME_SUB_BITS_BY_BUCKETS.items():
        xm = np.array([2 ** 31 - 1])
        assert O.log_bucket(xm, 10 ** 9, S)[0] <= nb - 1
        assert O.log_bucket(xm, 10 ** 9, S + 1)[0] > nb - 1


# ---------------------------------------------------------------- brute force
def test_bruteforce_tiny_workload():
    w = hw.tiny_fp32(0)
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    bf = np.array(BF.layer_bruteforce(w.X, w.offsets, w.timestamps, w.weights[0], w.dims))
    assert _relerr(ref, bf) < 1e-11


def test_bruteforce_edge_lengths_and_epochs():
    # an empty user, a length-1 user, unsorted timestamps and 64-bit epochs
    dims = _small_dims(n_pos_buckets=16, n_time_buckets=40, pos_sub_bits=1, time_sub_bits=1)
    w = hw.custom("edge", [0, 1, 7, 19, 3], dims, seed=3,
                  ts_base=[1_700_000_000, 1_600_000_000, 3, 1 << 40, 0])
    w.timestamps[5] += 5000   # one timestamp out of order
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    bf = np.array(BF.layer_bruteforce(w.X, w.offsets, w.timestamps, w.weights[0], w.dims))
    assert _relerr(ref, bf) < 1e-11


def test_padded_equals_jagged():
    dims = _small_dims()
    w = hw.custom("pad", [5, 1, 12, 0, 9], dims, seed=5)
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    pad = BF.layer_padded(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    assert _relerr(ref, pad) < 1e-12


def test_layer_rows_matches_full_layer():
    dims = _small_dims()
    w = hw.custom("rows", [40, 33], dims, seed=8)
    full = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    s, e = int(w.offsets[1]), int(w.offsets[2])
    rows = np.array([0, 5, 32])
    part, _ = O.layer_rows(w.X[s:e], w.timestamps[s:e], w.weights[0], dims, rows)
    assert np.allclose(part, full[s + rows], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- invariants
def test_causality_exact():
    dims = _small_dims()
    w = hw.custom("causal", [30, 25], dims, seed=11)
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    X2 = w.X.copy(); t2 = w.timestamps.copy()
    cut = 12                                  # perturb user 0 rows > cut
    X2[cut + 1:30] += 3.0
    t2[cut + 1:30] += 10_000
    got = O.layer_fwd(X2, w.offsets, t2, w.weights[0], w.dims)
    assert np.array_equal(got[:cut + 1], ref[:cut + 1])
    assert np.array_equal(got[30:], ref[30:])          # other user untouched
    assert not np.allclose(got[cut + 1:30], ref[cut + 1:30])


def test_one_over_n_linear():
    dims = _small_dims()
    w = hw.custom("norm", [17, 9], dims, seed=12)
    _, i1 = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims, return_intermediates=True)
    _, i2 = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims,
                        norm_len=[34, 18], return_intermediates=True)
    assert np.allclose(i2["O"] * 2.0, i1["O"], rtol=1e-13, atol=0)


def test_stack_is_layer_composition():
    dims = _small_dims()
    w = hw.custom("stack", [6, 11], dims, n_layers=3, seed=13)
    y = w.X.astype(np.float64)
    for lw in w.weights:
        y = O.layer_fwd(y, w.offsets, w.timestamps, lw, dims)
    assert np.array_equal(O.stack_fwd(w.X, w.offsets, w.timestamps, w.weights, dims), y)


# ---------------------------------------------------------------- special cases
def test_single_token_closed_form():
    dims = _small_dims()
    w = hw.custom("one", [1], dims, seed=14)
    lw = w.weights[0]
    _, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, lw, dims, return_intermediates=True)
    x = w.X[0].astype(np.float64)
    g = (x @ lw["W1"].T.astype(np.float64)) + lw["b1"].astype(np.float64)
    g = g / (1.0 + np.exp(-g))
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    for k in range(h):
        q = g[2 * h * dv + k * dqk: 2 * h * dv + (k + 1) * dqk]
        kk = g[2 * h * dv + h * dqk + k * dqk: 2 * h * dv + h * dqk + (k + 1) * dqk]
        v = g[h * dv + k * dv: h * dv + (k + 1) * dv]
        s = float(q @ kk) + float(lw["rab_pos"][k][0]) + float(lw["rab_time"][k][0])
        a = s / (1.0 + math.exp(-s))
        assert np.allclose(inter["O"][0, k * dv:(k + 1) * dv], a * v, rtol=1e-13, atol=1e-15)


def test_zero_values_give_beta_gate():
    dims = _small_dims()
    w = hw.custom("v0", [8, 5], dims, seed=15)
    lw = copy.deepcopy(w.weights[0])
    h, dv = dims.n_heads, dims.d_v
    lw["W1"][h * dv:2 * h * dv] = 0.0
    lw["b1"][h * dv:2 * h * dv] = 0.0
    Y, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, lw, dims, return_intermediates=True)
    X = w.X.astype(np.float64)
    expect = X + (lw["ln_beta"].astype(np.float64) * inter["U"]) @ lw["W2"].T.astype(np.float64) + lw["b2"].astype(np.float64)
    assert np.allclose(Y, expect, rtol=1e-12, atol=1e-12)


def test_zero_qk_leaves_rab_only():
    dims = _small_dims()
    w = hw.custom("qk0", [13], dims, seed=16)
    lw = copy.deepcopy(w.weights[0])
    h, dv, dqk = dims.n_heads, dims.d_v, dims.d_qk
    lw["W1"][2 * h * dv:] = 0.0
    lw["b1"][2 * h * dv:] = 0.0
    _, inter = O.layer_fwd(w.X, w.offsets, w.timestamps, lw, dims, return_intermediates=True)
    # Q = K = SiLU(0) = 0, so each score is the relative bias alone
    n = 13
    t = w.timestamps
    V = inter["V"]
    for k in range(h):
        for i in range(n):
            acc = np.zeros(dv)
            for j in range(i + 1):
                s = (float(lw["rab_pos"][k][BF.bucket_scalar(i - j, 32, 2)])
                     + float(lw["rab_time"][k][BF.bucket_scalar(max(0, int(t[i] - t[j])), 32, 0)]))
                acc += s / (1.0 + math.exp(-s)) * V[j, k * dv:(k + 1) * dv]
            assert np.allclose(inter["O"][i, k * dv:(k + 1) * dv], acc / n, rtol=1e-12, atol=1e-15)


def test_layer_norm_matches_torch_and_textbook():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    x = rng.normal(0.3, 2.0, size=(7, 48))
    g = rng.normal(1.0, 0.1, size=48); b = rng.normal(0.0, 0.1, size=48)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (48,), torch.from_numpy(g),
                                         torch.from_numpy(b), eps=1e-6).numpy()
    assert np.allclose(O.layer_norm(x, g, b, 1e-6), ref, rtol=1e-12, atol=1e-12)
    y = O.layer_norm(x, np.ones(48), np.zeros(48), 1e-6)
    v = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    assert np.allclose(y.var(axis=1), v / (v + 1e-6), rtol=1e-12)


def test_silu_matches_torch():
    torch = pytest.importorskip("torch")
    x = np.linspace(-60, 60, 2001)
    assert np.allclose(O.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                       rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------- M-FALCON
def _mf_workload(seed=21, n_layers=2):
    dims = _small_dims(n_pos_buckets=32, n_time_buckets=32, pos_sub_bits=2, time_sub_bits=0)
    return hw.custom("mf", [9, 14, 1], dims, n_layers=n_layers, seed=seed,
                     cands_per_user=[5, 7, 3], microbatch=3)


def _mf_scores(w, microbatch=None, cand_X=None, cand_offsets=None):
    return O.mfalcon_rank(w.X, w.offsets, w.timestamps,
                          w.candidates if cand_X is None else cand_X,
                          w.cand_offsets if cand_offsets is None else cand_offsets,
                          w.request_ts, w.microbatch if microbatch is None else microbatch,
                          w.head_vec, w.weights, w.dims)


def test_mfalcon_equals_naive_append():
    """The shared-history computation gives exactly what appending one
    candidate after the history and rerunning the whole stack gives."""
    w = _mf_workload()
    got = _mf_scores(w)
    for b in range(w.B):
        hs, he = int(w.offsets[b]), int(w.offsets[b + 1])
        cs, ce = int(w.cand_offsets[b]), int(w.cand_offsets[b + 1])
        n = he - hs
        for c in range(cs, ce):
            Xs = np.concatenate([w.X[hs:he], w.candidates[c:c + 1]])
            ts = np.concatenate([w.timestamps[hs:he], [w.request_ts[b]]])
            Y = O.stack_fwd(Xs, np.array([0, n + 1]), ts, w.weights, w.dims, norm_len=[n])
            naive = float(Y[-1] @ w.head_vec.astype(np.float64))
            assert abs(naive - got[c]) <= 1e-11 * max(1.0, abs(naive))


def test_mfalcon_microbatch_independent():
    w = _mf_workload()
    ref = _mf_scores(w, microbatch=1)
    for mb in (2, 3, 7, 100):
        assert np.allclose(_mf_scores(w, microbatch=mb), ref, rtol=1e-12, atol=1e-12)


def test_mfalcon_candidate_permutation_and_drop():
    w = _mf_workload()
    ref = _mf_scores(w)
    # permute user 1's candidates
    cs, ce = int(w.cand_offsets[1]), int(w.cand_offsets[2])
    perm = np.arange(len(w.candidates))
    perm[cs:ce] = perm[cs:ce][::-1]
    got = _mf_scores(w, cand_X=w.candidates[perm])
    assert np.allclose(got, ref[perm], rtol=1e-12, atol=1e-12)
    # drop all but one candidate of user 1
    keep = np.r_[0:cs, cs + 2, ce:len(w.candidates)]
    m = np.diff(w.cand_offsets).copy(); m[1] = 1
    off = np.concatenate([[0], np.cumsum(m)])
    got = _mf_scores(w, cand_X=w.candidates[keep], cand_offsets=off)
    assert np.allclose(got, ref[keep], rtol=1e-12, atol=1e-12)


def test_mfalcon_empty_history_single_candidate_closed_form():
    # With no history the candidate attends only to itself: one layer reduces
    # to o = SiLU(q.k + Rp[0] + Rt[0]) v / max(n,1) with n = 0 -> 1.
    dims = _small_dims()
    w = hw.custom("mf0", [0], dims, n_layers=1, seed=22, cands_per_user=[1])
    lw = w.weights[0]
    s = O.mfalcon_rank(w.X, w.offsets, w.timestamps, w.candidates, w.cand_offsets,
                       np.array([0]), 1, w.head_vec, w.weights, dims)[0]
    x = w.candidates[0].astype(np.float64)
    g = x @ lw["W1"].T.astype(np.float64) + lw["b1"].astype(np.float64)
    g = g / (1 + np.exp(-g))
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    o = np.zeros(h * dv)
    for k in range(h):
        q = g[2 * h * dv + k * dqk:2 * h * dv + (k + 1) * dqk]
        kk = g[2 * h * dv + h * dqk + k * dqk:2 * h * dv + h * dqk + (k + 1) * dqk]
        sc = float(q @ kk) + float(lw["rab_pos"][k][0]) + float(lw["rab_time"][k][0])
        o[k * dv:(k + 1) * dv] = sc / (1 + math.exp(-sc)) * g[h * dv + k * dv:h * dv + (k + 1) * dv]
    mu, var = o.mean(), o.var()
    z = ((o - mu) / math.sqrt(var + dims.ln_eps) * lw["ln_gamma"].astype(np.float64)
         + lw["ln_beta"].astype(np.float64)) * g[:h * dv]
    y = x + z @ lw["W2"].T.astype(np.float64) + lw["b2"].astype(np.float64)
    assert abs(float(y @ w.head_vec.astype(np.float64)) - s) < 1e-12


# ---------------------------------------------------------------- planted mistakes
def _pins_hold():
    """The cheap pins a planted mistake must break (brute force, M-FALCON)."""
    dims = _small_dims(n_pos_buckets=16, n_time_buckets=40, pos_sub_bits=1, time_sub_bits=1)
    w = hw.custom("plant", [0, 1, 7, 11], dims, seed=31)
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], w.dims)
    bf = np.array(BF.layer_bruteforce(w.X, w.offsets, w.timestamps, w.weights[0], w.dims))
    ok = _relerr(ref, bf) < 1e-11
    wm = _mf_workload(seed=32, n_layers=1)
    got = _mf_scores(wm)
    b, c = 1, int(wm.cand_offsets[1])
    hs, he = int(wm.offsets[b]), int(wm.offsets[b + 1])
    Xs = np.concatenate([wm.X[hs:he], wm.candidates[c:c + 1]])
    ts = np.concatenate([wm.timestamps[hs:he], [wm.request_ts[b]]])
    Y = O.stack_fwd(Xs, np.array([0, he - hs + 1]), ts, wm.weights, wm.dims, norm_len=[he - hs])
    ok = ok and abs(float(Y[-1] @ wm.head_vec) - got[c]) < 1e-11
    return ok


@pytest.mark.parametrize("mistake", ["swap_qk", "drop_time_bias", "bucket_off_by_one",
                                     "sigmoid_not_silu", "ln_no_center", "norm_n_plus_1",
                                     "split_v_u"])
def test_planted_mistake_is_caught(monkeypatch, mistake):
    assert _pins_hold()
    if mistake == "swap_qk":
        orig = O.split_uvqk
        monkeypatch.setattr(O, "split_uvqk", lambda G, d: {**orig(G, d), "Q": orig(G, d)["K"],
                                                           "K": orig(G, d)["Q"]})
    elif mistake == "split_v_u":
        orig = O.split_uvqk
        monkeypatch.setattr(O, "split_uvqk", lambda G, d: {**orig(G, d), "U": orig(G, d)["V"],
                                                           "V": orig(G, d)["U"]})
    elif mistake == "drop_time_bias":
        orig = O._attention_user

        def no_time(Q, K, V, t, w, dims, norm, rows=None):
            w2 = dict(w); w2["rab_time"] = np.zeros_like(w["rab_time"])
            return orig(Q, K, V, t, w2, dims, norm, rows)
        monkeypatch.setattr(O, "_attention_user", no_time)
    elif mistake == "bucket_off_by_one":
        orig = O.log_bucket
        monkeypatch.setattr(O, "log_bucket", lambda x, n, s: np.minimum(orig(x, n, s) + 1, n - 1))
    elif mistake == "sigmoid_not_silu":
        monkeypatch.setattr(O, "silu", lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64))))
    elif mistake == "ln_no_center":
        monkeypatch.setattr(O, "layer_norm",
                            lambda x, g, b, e: x / np.sqrt((x ** 2).mean(-1, keepdims=True) + e) * g + b)
    elif mistake == "norm_n_plus_1":
        orig = O._attention_user
        monkeypatch.setattr(O, "_attention_user",
                            lambda Q, K, V, t, w, dims, norm, rows=None: orig(Q, K, V, t, w, dims, norm + 1, rows))
    assert not _pins_hold()
