"""GPU parity of Stochastic Length sampling + token embedding (hstu_sl_embed,
through the C ABI) against the oracle (oracle.stochastic_length) on the same
seeded raw streams.

Everything here is integer or byte work, so the bar is bit-exact: the kept
offsets, the kept timestamps and every bf16 embedding row (compared as bit
patterns) must equal the oracle's.  Status checks: offsets that do not
describe the raw batch set HSTU_ERR_BAD_OFFSETS (all kept offsets 0); an id
outside its table sets HSTU_ERR_BAD_IDS and zeroes that row only.
"""
import numpy as np
import pytest

import hstu_workloads as hw
from oracle import stochastic_length as SL

pytestmark = pytest.mark.gpu

HSTU_OK, HSTU_ERR_UNSUPPORTED, HSTU_ERR_BAD_OFFSETS, HSTU_ERR_BAD_IDS = 0, 2, 5, 8


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _bits_to_device(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run(rs, ctab, atab, raw_offsets=None, raw_ids=None):
    """Runs hstu_sl_embed; returns (status, offsets, X bits uint16 [T, d], ts)."""
    import torch
    import hstu_sequential_transducer_layer_b200 as H
    from hstu_sequential_transducer_layer_b200 import binding as Bd
    off = raw_offsets if raw_offsets is not None else rs.raw_offsets
    ids = raw_ids if raw_ids is not None else rs.raw_ids
    B, R, d = len(off) - 1, rs.R, rs.d_model
    dev = torch.device("cuda")
    t_off = torch.from_numpy(np.asarray(off, np.int64)).to(dev)
    t_ids = torch.from_numpy(np.asarray(ids, np.int64)).to(dev)
    t_ts = torch.from_numpy(rs.raw_timestamps).to(dev)
    out_off = torch.full((B + 1,), -1, dtype=torch.int64, device=dev)
    X = torch.full((max(R, 1), d), float("nan"), dtype=torch.bfloat16, device=dev)
    out_ts = torch.full((max(R, 1),), -1, dtype=torch.int64, device=dev)
    ws = torch.empty(Bd.hstu_sl_embed_workspace_size(), dtype=torch.uint8, device=dev)
    Bd.hstu_sl_embed(B, R, rs.max_raw_len, t_off, t_ids, t_ts, rs.sl_seed, ctab, atab, out_off, X,
                     out_ts, ws)
    st = H.hstu_read_status(ws)
    o = out_off.cpu().numpy()
    T = int(o[-1]) if st == HSTU_OK or st == HSTU_ERR_BAD_IDS else 0
    xb = X[:T].view(torch.int16).cpu().numpy().view(np.uint16)
    return st, o, xb, out_ts[:T].cpu().numpy()


def _check(rs, cbits, abits, ctab=None, atab=None):
    ctab = ctab if ctab is not None else _bits_to_device(cbits)
    atab = atab if atab is not None else _bits_to_device(abits)
    st, o, xb, ts = _run(rs, ctab, atab)
    assert st == HSTU_OK, st
    ref_o, ref_x, ref_ts = SL.sl_embed(rs.raw_offsets, rs.raw_ids, rs.raw_timestamps, rs.sl_seed,
                                       cbits, abits)
    np.testing.assert_array_equal(o, ref_o)
    np.testing.assert_array_equal(ts, ref_ts)
    assert xb.shape == ref_x.shape
    np.testing.assert_array_equal(xb.astype(np.float64), ref_x)
    return o


def _small(lengths, d=64, n_content=1000, n_actions=8, seed=0, **kw):
    rs = hw.raw_stream("sl_small", lengths, d, n_content, n_actions, seed=seed, **kw)
    return (rs, hw.embedding_table_bits(seed, 0, n_content, d),
            hw.embedding_table_bits(seed, 1, n_actions, d))


@pytest.mark.parametrize("d", [8, 64, 1024])
def test_edge_lengths_match_oracle(d):
    # empty users, a single token, two tokens, lengths around the 256-position
    # chunk of the compaction, and lengths whose keep count is 1
    lengths = [0, 1, 2, 3, 5, 0, 33, 255, 256, 257, 300, 513, 1000, 0]
    rs, c, a = _small(lengths, d=d, seed=d)
    o = _check(rs, c, a)
    assert [o[i + 1] - o[i] for i in range(len(lengths))] == [SL.keep_count(n) for n in lengths]


def test_long_users_and_keep_count_extremes():
    # the maximum supported raw length (32767) and values at which floor(n^0.8)
    # steps; the kept offsets test the device keep count against the oracle's
    lengths = [32767, 32766, 16384, 4096, 4095, 3125, 3124, 1024, 243, 32, 31, 1]
    rs, c, a = _small(lengths, d=16, n_content=5000, seed=7, max_raw_len=32767)
    _check(rs, c, a)


def test_many_users_more_than_one_wave():
    rng = np.random.default_rng(11)
    lengths = rng.integers(0, 600, size=1500)
    rs, c, a = _small(lengths, d=32, n_content=20000, seed=11)
    _check(rs, c, a)


def test_more_users_than_one_block_can_offset():
    # beyond 2048 users the kept offsets come from their own kernel
    rng = np.random.default_rng(12)
    lengths = rng.integers(0, 60, size=2500)
    rs, c, a = _small(lengths, d=8, n_content=500, seed=12)
    _check(rs, c, a)


def test_empty_batch_and_all_empty_users():
    for lengths in ([], [0, 0, 0]):
        rs, c, a = _small(lengths, d=64, seed=3)
        st, o, xb, ts = _run(rs, _bits_to_device(c), _bits_to_device(a))
        assert st == HSTU_OK
        np.testing.assert_array_equal(o, np.zeros(len(lengths) + 1, np.int64))


def test_seed_changes_selection():
    rs, c, a = _small([4096], d=8, seed=5)
    o1 = _check(rs, c, a)
    rs.sl_seed ^= 1
    o2 = _check(rs, c, a)
    np.testing.assert_array_equal(o1, o2)
    k1 = SL.kept_positions(rs.sl_seed ^ 1, 0, 4096)
    k2 = SL.kept_positions(rs.sl_seed, 0, 4096)
    assert not np.array_equal(k1, k2)


def test_full_stack_raw_at_full_size():
    """The raw input of the 8-layer stack workload at its full size (B=128,
    lognormal raw lengths up to 4096, d=1024, a 1M-row content table), in the
    launch configuration the benchmark times."""
    rs = hw.full_stack_raw(0)
    ctab = hw.device_embedding_table(0, 0, rs.n_content, rs.d_model, "cuda")
    atab = hw.device_embedding_table(0, 1, rs.n_actions, rs.d_model, "cuda")
    import torch
    cbits = ctab.view(torch.int16).cpu().numpy().view(np.uint16)
    abits = atab.view(torch.int16).cpu().numpy().view(np.uint16)
    o = _check(rs, cbits, abits, ctab, atab)
    assert o[-1] > 0 and max(np.diff(o)) <= SL.keep_count(4096)


def test_bad_offsets_set_status():
    rs, c, a = _small([10, 20, 30], d=16, seed=2)
    ct, at = _bits_to_device(c), _bits_to_device(a)
    bad = [
        np.array([1, 10, 30, 60]),        # does not start at 0
        np.array([0, 20, 10, 60]),        # decreasing
        np.array([0, 10, 30, 59]),        # does not end at the raw total
    ]
    for off in bad:
        st, o, _, _ = _run(rs, ct, at, raw_offsets=off)
        assert st == HSTU_ERR_BAD_OFFSETS, (off, st)
        np.testing.assert_array_equal(o, np.zeros(4, np.int64))
    # no users but a nonzero raw total
    st, o, _, _ = _run(rs, ct, at, raw_offsets=np.array([0]))
    assert st == HSTU_ERR_BAD_OFFSETS and o.tolist() == [0]
    # a batch larger than the single-block offsets path, one length negative
    rs_big, cb, ab = _small(np.full(2100, 3), d=16, seed=4)
    off = rs_big.raw_offsets.copy()
    off[1000] = off[1002]
    st, o, _, _ = _run(rs_big, _bits_to_device(cb), _bits_to_device(ab), raw_offsets=off)
    assert st == HSTU_ERR_BAD_OFFSETS
    np.testing.assert_array_equal(o, np.zeros(2101, np.int64))
    # a user longer than max_raw_len
    rs.max_raw_len = 25
    st, o, _, _ = _run(rs, ct, at)
    assert st == HSTU_ERR_BAD_OFFSETS
    # max_raw_len above the supported bound is refused on the host
    from hstu_sequential_transducer_layer_b200 import HstuError
    rs.max_raw_len = 40000
    with pytest.raises(HstuError) as e:
        _run(rs, ct, at)
    assert e.value.code == HSTU_ERR_UNSUPPORTED


def test_bad_id_sets_status_and_zeroes_its_row():
    # user 1 has one token (always kept, position 0 = content): give it an id
    # one past the end of the content table
    rs, c, a = _small([50, 1, 70], d=64, n_content=100, seed=9)
    ids = rs.raw_ids.copy()
    ids[50] = 100
    st, o, xb, ts = _run(rs, _bits_to_device(c), _bits_to_device(a), raw_ids=ids)
    assert st == HSTU_ERR_BAD_IDS
    ref_o, ref_x, ref_ts = SL.sl_embed(rs.raw_offsets, rs.raw_ids, rs.raw_timestamps, rs.sl_seed,
                                       c, a)
    np.testing.assert_array_equal(o, ref_o)
    np.testing.assert_array_equal(ts, ref_ts)
    bad_row = int(ref_o[1])
    assert not xb[bad_row].any()
    keep = np.arange(len(ref_x)) != bad_row
    np.testing.assert_array_equal(xb[keep].astype(np.float64), ref_x[keep])


def _bits_to_f32(bits):
    return (np.asarray(bits, np.uint32) << np.uint32(16)).view(np.float32)


def test_pipeline_raw_streams_to_stack_matches_oracle():
    """Raw streams -> Stochastic Length + embedding -> 2-layer stack on the
    GPU (HSTURunner.stack_raw, no host synchronisation in between) against
    the oracle's sl_embed followed by its stack."""
    import torch
    from oracle import hstu_oracle as O
    from gpu_util import TOL, relerr, rmserr, runner_for
    dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
    w = hw.custom("pipe", [1], dims, n_layers=2, seed=50)
    rs, c, a = _small([2000, 1, 700, 0, 129, 4096], d=256, n_content=3000, seed=50)
    ref_o, ref_x, ref_ts = SL.sl_embed(rs.raw_offsets, rs.raw_ids, rs.raw_timestamps, rs.sl_seed,
                                       _bits_to_f32(c), _bits_to_f32(a))
    ref = O.stack_fwd(ref_x, ref_o, ref_ts, w.weights, dims)
    r = runner_for(w)
    dev = [torch.from_numpy(x).cuda() for x in (rs.raw_offsets, rs.raw_ids, rs.raw_timestamps)]
    out, off, ts = r.stack_raw(np.diff(rs.raw_offsets), *dev, rs.sl_seed, _bits_to_device(c),
                               _bits_to_device(a), rs.max_raw_len)
    torch.cuda.synchronize()
    assert r.sl_status() == HSTU_OK and r.status() == HSTU_OK
    np.testing.assert_array_equal(off.cpu().numpy(), ref_o)
    np.testing.assert_array_equal(ts.cpu().numpy(), ref_ts)
    Y = out.double().cpu().numpy()
    e, ed = relerr(Y, ref), rmserr(Y - ref_x, ref - ref_x)
    print("pipeline", e, ed)
    assert e <= TOL[hw.BF16] and ed <= TOL[hw.BF16]
