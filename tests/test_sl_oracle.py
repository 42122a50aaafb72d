"""Pins of the Stochastic Length + embedding oracle (oracle/stochastic_length.py)
against facts from outside it: the published SplitMix64 outputs, the page's
kept length 776 at 4096, the integer characterisation of floor(n^0.8), a
brute-force selection, and the selection's inclusion frequencies."""
import math
import os

import numpy as np

from oracle import stochastic_length as SL

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    out = []
    for line in open(os.path.join(HERE, "golden", "splitmix64.txt")):
        if line.strip() and not line.startswith("#"):
            i, h = line.split()
            out.append((int(i), int(h, 16)))
    return out


def test_splitmix64_matches_published_outputs():
    for i, v in _golden():
        assert SL.splitmix64_output(0, i) == v
    # position p of user 0 is output number p + 1
    k = SL.keys(0, 0, 2)
    assert [int(x) for x in k] == [v for _, v in _golden()]


def test_vectorised_generator_equals_scalar():
    rng = np.random.default_rng(0)
    seeds = [0, 1, 12345, 2**63 + 7]
    c = rng.integers(0, 2**40, size=200, dtype=np.int64).astype(np.uint64)
    for s in seeds:
        vec = SL.splitmix64_outputs(s, c)
        assert all(int(v) == SL.splitmix64_output(s, int(x)) for v, x in zip(vec, c))


def test_keep_count_closed_forms():
    # 'HSTUとGenerative Recommenders', section '2. Stochastic Lengthで学習時の履歴を間引く':
    # a 4096-token history is shortened to 776 tokens
    assert SL.keep_count(4096) == 776
    assert SL.keep_count(0) == 0 and SL.keep_count(1) == 1 and SL.keep_count(2) == 1
    for n in list(range(1, 3000)) + [3125, 4095, 4097, 32768, 65535]:
        k = SL.keep_count(n)
        assert k ** 5 <= n ** 4 < (k + 1) ** 5 or k == n  # k = floor(n^(4/5)), exactly
        assert k == min(n, math.floor(n ** 0.8))


def test_kept_positions_equal_brute_force_sort():
    for seed in (0, 7, 2**40 + 3):
        for b, n in ((0, 1), (1, 2), (3, 10), (5, 33), (9, 130)):
            keys = [SL.splitmix64_output(seed, (b << 32) + p + 1) for p in range(n)]
            k = SL.keep_count(n)
            brute = sorted(sorted(range(n), key=lambda p: (keys[p], p))[:k])
            got = SL.kept_positions(seed, b, n)
            assert list(got) == brute
            assert len(set(got)) == k and all(0 <= p < n for p in got)


def test_inclusion_frequencies_are_uniform():
    n, k = 10, SL.keep_count(10)  # 6 of 10
    counts = np.zeros(n)
    trials = 3000
    for seed in range(trials):
        counts[SL.kept_positions(seed, 3, n)] += 1
    freq = counts / trials
    assert np.all(np.abs(freq - k / n) < 0.04), freq


def test_sl_embed_alternates_tables_and_keeps_timestamps():
    rng = np.random.default_rng(1)
    lens = [0, 1, 5, 40]
    off = np.concatenate([[0], np.cumsum(lens)])
    ids = rng.integers(0, 6, size=off[-1])
    ts = np.arange(off[-1]) * 10 + 3
    ct = rng.normal(size=(6, 4))
    at = rng.normal(size=(6, 4)) + 100.0
    o, X, t = SL.sl_embed(off, ids, ts, 5, ct, at)
    assert list(np.diff(o)) == [SL.keep_count(n) for n in lens]
    row = 0
    for b, n in enumerate(lens):
        for p in SL.kept_positions(5, b, n):
            r = off[b] + p
            want = ct[ids[r]] if p % 2 == 0 else at[ids[r]]
            assert np.array_equal(X[row], want) and t[row] == ts[r]
            row += 1
    assert row == o[-1]
