"""Pure-Python brute force (explicit i, j, k loops) and a padded dense variant.

TEST INFRASTRUCTURE ONLY: these exist to pin ``hstu_oracle`` and are used by
``tests/`` alone.  They restate the same definitions ('HSTUとGenerative
Recommenders', section 'HSTUはTransformerと何が違うのか') with different
code: Python floats and loops, a bucket function that finds the exponent by
repeated shifting, and (for the padded variant) a dense [B, N_max] batch with
an explicit mask.  They share no helper with ``hstu_oracle``.
"""
from __future__ import annotations

import math
from typing import Dict, List

import numpy as np


def bucket_scalar(x: int, n_buckets: int, sub_bits: int) -> int:
    """Log-linear bucket by repeated shifting (no logarithms)."""
    assert x >= 0
    lim = 1 << sub_bits
    if x < lim:
        b = x
    else:
        e = 0
        y = x
        while y > 1:
            y >>= 1
            e += 1
        b = (e - sub_bits + 1) * lim + ((x >> (e - sub_bits)) - lim)
    return min(b, n_buckets - 1)


def _silu(v: float) -> float:
    if v >= 0:
        return v / (1.0 + math.exp(-v))
    ev = math.exp(v)
    return v * ev / (1.0 + ev)


def _dot(a, b) -> float:
    s = 0.0
    for x, y in zip(a, b):
        s += x * y
    return s


def layer_bruteforce(X, offsets, timestamps, w: Dict[str, np.ndarray], dims) -> List[List[float]]:
    """One layer with every sum written as a Python loop.  Returns rows of Y."""
    h, dqk, dv, d = dims.n_heads, dims.d_qk, dims.d_v, dims.d_model
    F = 2 * h * dv + 2 * h * dqk
    W1 = w["W1"].astype(float).tolist(); b1 = w["b1"].astype(float).tolist()
    W2 = w["W2"].astype(float).tolist(); b2 = w["b2"].astype(float).tolist()
    gam = w["ln_gamma"].astype(float).tolist(); bet = w["ln_beta"].astype(float).tolist()
    Rp = w["rab_pos"].astype(float).tolist(); Rt = w["rab_time"].astype(float).tolist()
    Xl = np.asarray(X, dtype=np.float64).tolist()
    ts = [int(v) for v in timestamps]
    T = len(Xl)
    # f1 + SiLU, per token
    G = []
    for i in range(T):
        G.append([_silu(_dot(W1[f], Xl[i]) + b1[f]) for f in range(F)])
    uo, vo, qo, ko = 0, h * dv, 2 * h * dv, 2 * h * dv + h * dqk
    Y = [None] * T
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        for i in range(s, e):
            o = [0.0] * (h * dv)
            for k in range(h):
                for j in range(s, i + 1):
                    q = G[i][qo + k * dqk: qo + (k + 1) * dqk]
                    kk = G[j][ko + k * dqk: ko + (k + 1) * dqk]
                    sc = _dot(q, kk)
                    sc += Rp[k][bucket_scalar(i - j, dims.n_pos_buckets, dims.pos_sub_bits)]
                    sc += Rt[k][bucket_scalar(max(0, ts[i] - ts[j]), dims.n_time_buckets,
                                              dims.time_sub_bits)]
                    a = _silu(sc)
                    for c in range(dv):
                        o[k * dv + c] += a * G[j][vo + k * dv + c]
            o = [x / n for x in o]
            mu = sum(o) / len(o)
            var = sum((x - mu) ** 2 for x in o) / len(o)
            rs = 1.0 / math.sqrt(var + dims.ln_eps)
            z = [((o[c] - mu) * rs * gam[c] + bet[c]) * G[i][uo + c] for c in range(h * dv)]
            Y[i] = [Xl[i][r] + _dot(W2[r], z) + b2[r] for r in range(d)]
    return Y


def layer_padded(X, offsets, timestamps, w, dims) -> np.ndarray:
    """Dense padded batch [B, N_max, .] with mask j <= i < n_b and normaliser
    n_b; the jagged result must equal this one row for row."""
    offsets = np.asarray(offsets, np.int64)
    B = len(offsets) - 1
    lens = np.diff(offsets)
    N = int(lens.max()) if B else 0
    d, h, dqk, dv = dims.d_model, dims.n_heads, dims.d_qk, dims.d_v
    Xp = np.zeros((B, N, d)); tp = np.zeros((B, N), np.int64)
    for b in range(B):
        Xp[b, :lens[b]] = X[offsets[b]:offsets[b + 1]]
        tp[b, :lens[b]] = timestamps[offsets[b]:offsets[b + 1]]
    W1 = w["W1"].astype(np.float64); W2 = w["W2"].astype(np.float64)
    pre = np.einsum("bnd,fd->bnf", Xp, W1) + w["b1"]
    G = pre * (1.0 / (1.0 + np.exp(-pre)))
    U = G[..., :h * dv]; V = G[..., h * dv:2 * h * dv]
    Q = G[..., 2 * h * dv:2 * h * dv + h * dqk]; K = G[..., 2 * h * dv + h * dqk:]
    ii = np.arange(N)[:, None]; jj = np.arange(N)[None, :]
    valid = (jj <= ii)[None] & (ii < lens[:, None, None])
    bpos = np.vectorize(lambda x: bucket_scalar(int(x), dims.n_pos_buckets, dims.pos_sub_bits))(
        np.maximum(ii - jj, 0))
    gap = np.maximum(tp[:, :, None] - tp[:, None, :], 0)
    btime = np.vectorize(lambda x: bucket_scalar(int(x), dims.n_time_buckets, dims.time_sub_bits))(gap)
    O = np.zeros((B, N, h * dv))
    for k in range(h):
        Qk = Q[..., k * dqk:(k + 1) * dqk]; Kk = K[..., k * dqk:(k + 1) * dqk]
        Vk = V[..., k * dv:(k + 1) * dv]
        sc = np.einsum("bic,bjc->bij", Qk, Kk) + w["rab_pos"][k][bpos][None] + w["rab_time"][k][btime]
        A = np.where(valid, sc / (1.0 + np.exp(-sc)), 0.0)
        O[..., k * dv:(k + 1) * dv] = np.einsum("bij,bjc->bic", A, Vk) / np.maximum(lens, 1)[:, None, None]
    mu = O.mean(-1, keepdims=True)
    var = O.var(-1, keepdims=True)
    Z = ((O - mu) / np.sqrt(var + dims.ln_eps) * w["ln_gamma"] + w["ln_beta"]) * U
    Yp = Xp + np.einsum("bnc,dc->bnd", Z, W2) + w["b2"]
    return np.concatenate([Yp[b, :lens[b]] for b in range(B)], axis=0) if B else np.zeros((0, d))
