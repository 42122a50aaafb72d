"""Oracle for Stochastic Length sampling and token embedding (test
infrastructure only: the GPU path never imports this module).

Source: 'HSTUとGenerative Recommenders', section '2. Stochastic Lengthで学習時の
履歴を間引く' (a long history is shortened to a random subset of its positions;
with the 4096 cap and alpha 1.6 the typical kept length is 776), read as:

* keep count k = min(n, floor(n ** 0.8)), at least 1 for n >= 1 (the keep
  fraction that maps 4096 to 776);
* the kept positions are a uniformly random k-subset of 0..n-1 in their
  original order: every position gets a 64-bit key and the k smallest keys
  (ties by position) are kept;
* keys are counter-based so that any implementation reproduces them: the key
  of position p of user b is output number b * 2**32 + p + 1 of the SplitMix64
  generator (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014) started from state `seed`;
* token embeddings: a token at an even original position is a content item
  (row `id` of the content table), at an odd position an action (row `id` of
  the action table) -- content and action tokens alternate in the raw stream;
  timestamps are those of the kept tokens.

Plain numpy; integers throughout (no rounding can differ between sides).
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def splitmix64_output(seed: int, i: int) -> int:
    """Output number i (1-based) of SplitMix64 started from state `seed`:
    the state advances by the golden-ratio increment, and each state is
    mixed by two xor-shift-multiply rounds and a final xor-shift."""
    z = (seed + i * GAMMA) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64_outputs(seed: int, counters: np.ndarray) -> np.ndarray:
    """Vectorised splitmix64_output(seed, counters) on uint64 (wrapping)."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed & MASK64) + counters.astype(np.uint64) * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def keep_count(n: int) -> int:
    """min(n, floor(n ** 0.8)), at least 1 (0 for an empty sequence); exact:
    the largest k with k**5 <= n**4."""
    if n <= 0:
        return 0
    k = int(round(n ** 0.8))
    while k ** 5 > n ** 4:
        k -= 1
    while (k + 1) ** 5 <= n ** 4:
        k += 1
    return max(1, min(n, k))


def keys(seed: int, b: int, n: int) -> np.ndarray:
    """The 64-bit keys of positions 0..n-1 of user b."""
    c = (np.uint64(b) << np.uint64(32)) + np.arange(n, dtype=np.uint64) + np.uint64(1)
    return splitmix64_outputs(seed, c)


def kept_positions(seed: int, b: int, n: int) -> np.ndarray:
    """Positions kept for user b (sorted): the keep_count(n) smallest keys,
    ties broken by position."""
    k = keep_count(n)
    if k == 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((np.arange(n), keys(seed, b, n)))
    return np.sort(order[:k]).astype(np.int64)


def sl_embed(raw_offsets, raw_ids, raw_ts, seed, content_table, action_table):
    """Stochastic Length + embedding for a jagged batch.

    Returns (offsets [B+1] int64, X [T, d] float64, timestamps [T] int64)."""
    raw_offsets = np.asarray(raw_offsets, np.int64)
    B = len(raw_offsets) - 1
    offs = [0]
    rows, ts = [], []
    for b in range(B):
        r0, r1 = int(raw_offsets[b]), int(raw_offsets[b + 1])
        pos = kept_positions(seed, b, r1 - r0)
        for p in pos:
            i = int(raw_ids[r0 + p])
            rows.append(content_table[i] if p % 2 == 0 else action_table[i])
            ts.append(int(raw_ts[r0 + p]))
        offs.append(offs[-1] + len(pos))
    d = content_table.shape[1]
    X = np.asarray(rows, np.float64).reshape(len(rows), d)
    return np.asarray(offs, np.int64), X, np.asarray(ts, np.int64)
