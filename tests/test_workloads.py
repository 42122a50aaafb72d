"""The seeded input generators: determinism, shapes, storage rounding, and the
Stochastic Length keep rule."""
import math

import numpy as np
import pytest

import hstu_workloads as hw


def test_stochastic_length_776():
    # the typical shortened length quoted for max length 4096 (4096^0.8 = 776.05)
    assert hw.stochastic_length_keep(4096) == 776
    assert 4096 ** 0.8 == pytest.approx(776.047, abs=1e-3)
    assert hw.stochastic_length_keep(2) == 1
    assert hw.stochastic_length_keep(1) == 1
    for n in (3, 10, 100, 1000, 4095):
        k = hw.stochastic_length_keep(n)
        assert 1 <= k <= n and k == min(n, math.floor(n ** 0.8))


def test_round_to_bf16_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.normal(0, 1, 10000), rng.normal(0, 1e-30, 100),
                        [0.0, -0.0, 1.0, 65504.0, 3.4e38]]).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(hw.round_to_bf16(a), ref)


def test_tiny_deterministic_and_shaped():
    a, b = hw.tiny_fp32(0), hw.tiny_fp32(0)
    assert np.array_equal(a.X, b.X) and np.array_equal(a.offsets, b.offsets)
    assert a.B == 4 and a.dims.d_model == 64 and a.dims.dtype == hw.FP32
    assert all(8 <= n <= 64 for n in a.lengths)
    assert a.timestamps.dtype == np.int64 and a.timestamps.shape == (a.T,)
    for bb in range(a.B):
        t = a.timestamps[a.offsets[bb]:a.offsets[bb + 1]]
        assert t[0] == 0 and np.all(np.diff(t) >= 0)
    c = hw.tiny_fp32(1)
    assert not np.array_equal(a.X[:8], c.X[:8])


def test_single_layer_lengths_and_bf16():
    w = hw.single_layer(0)
    assert w.B == 64 and w.lengths.max() <= 1024 and w.lengths.min() >= 1
    assert np.array_equal(hw.round_to_bf16(w.X), w.X)
    assert np.array_equal(hw.round_to_bf16(w.weights[0]["W1"]), w.weights[0]["W1"])
    assert w.weights[0]["W1"].shape == (w.dims.f1_width, 256)
    assert w.weights[0]["W2"].shape == (256, 256)
    assert w.weights[0]["rab_pos"].shape == (4, 128)


def test_mfalcon_small_shapes():
    w = hw.mfalcon(0, n_users=3, cands=10, microbatch=4)
    assert w.n_layers == 3 and w.candidates.shape == (30, 512)
    assert np.array_equal(w.cand_offsets, [0, 10, 20, 30])
    assert w.request_ts.shape == (3,)
    for b in range(3):
        assert w.request_ts[b] == w.timestamps[w.offsets[b + 1] - 1]


@pytest.mark.slow
def test_full_stack_shape_small():
    w = hw.full_stack(0, n_users=6)
    assert w.n_layers == 8 and w.max_len == 776
    raw = w.meta["raw_lengths"]
    assert np.array_equal(w.lengths, [hw.stochastic_length_keep(int(n)) for n in raw])
    assert np.array_equal(hw.round_to_bf16(w.X), w.X)
