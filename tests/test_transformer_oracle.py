"""Pins of the softmax-Transformer comparator's oracle (oracle.transformer):
pure-Python loops on a tiny case, torch's causal scaled-dot-product attention,
closed forms (uniform weights, one token), row sums, causality, and planted
mistakes."""
import math

import numpy as np
import torch

from oracle import transformer as TR


def _weights(rng, d, heads, ff):
    s = 1.0 / math.sqrt(d)
    return dict(ln1_gamma=1 + 0.1 * rng.normal(size=d), ln1_beta=0.1 * rng.normal(size=d),
                W_qkv=s * rng.normal(size=(3 * d, d)), W_o=s * rng.normal(size=(d, d)),
                ln2_gamma=1 + 0.1 * rng.normal(size=d), ln2_beta=0.1 * rng.normal(size=d),
                W_1=s * rng.normal(size=(ff, d)), b_1=0.1 * rng.normal(size=ff),
                W_2=(1 / math.sqrt(ff)) * rng.normal(size=(d, ff)), b_2=0.1 * rng.normal(size=d))


def _loops(X, w, heads, eps):
    """The layer with explicit loops over positions, heads and features."""
    n, d = X.shape
    dh = d // heads

    def ln(x, g, b):
        mu = sum(x) / len(x)
        var = sum((v - mu) ** 2 for v in x) / len(x)
        return [(x[k] - mu) / math.sqrt(var + eps) * g[k] + b[k] for k in range(len(x))]

    def mat(Wm, x):
        return [sum(Wm[o][k] * x[k] for k in range(len(x))) for o in range(len(Wm))]

    A = [ln(list(X[i]), w["ln1_gamma"], w["ln1_beta"]) for i in range(n)]
    QKV = [mat(w["W_qkv"], A[i]) for i in range(n)]
    ctx = [[0.0] * d for _ in range(n)]
    for h in range(heads):
        for i in range(n):
            sc = []
            for j in range(i + 1):
                sc.append(sum(QKV[i][h * dh + c] * QKV[j][d + h * dh + c] for c in range(dh))
                          / math.sqrt(dh))
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            tot = sum(ex)
            for c in range(dh):
                ctx[i][h * dh + c] = sum(ex[j] / tot * QKV[j][2 * d + h * dh + c]
                                         for j in range(i + 1))
    Y = []
    for i in range(n):
        o = mat(w["W_o"], ctx[i])
        x1 = [X[i][k] + o[k] for k in range(d)]
        b = ln(x1, w["ln2_gamma"], w["ln2_beta"])
        f = [v + w["b_1"][k] for k, v in enumerate(mat(w["W_1"], b))]
        f = [v / (1 + math.exp(-v)) for v in f]
        y = [x1[k] + v + w["b_2"][k] for k, v in enumerate(mat(w["W_2"], f))]
        Y.append(y)
    return np.array(Y)


def test_matches_loops():
    rng = np.random.default_rng(0)
    d, heads, ff, n = 8, 2, 16, 6
    w = _weights(rng, d, heads, ff)
    X = rng.normal(size=(n, d))
    np.testing.assert_allclose(TR.user_fwd(X, w, heads, 1e-6), _loops(X, w, heads, 1e-6),
                               rtol=0, atol=1e-12)


def test_attention_matches_torch_causal_sdpa():
    rng = np.random.default_rng(1)
    n, heads, dh = 37, 4, 16
    Q, K, V = (rng.normal(size=(n, heads * dh)) for _ in range(3))
    ours = TR.attention(Q, K, V, heads)
    t = [torch.from_numpy(M).reshape(n, heads, dh).transpose(0, 1) for M in (Q, K, V)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True)
    np.testing.assert_allclose(ours, ref.transpose(0, 1).reshape(n, heads * dh).numpy(),
                               rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one_and_respect_the_mask():
    rng = np.random.default_rng(2)
    P = TR.softmax_causal(rng.normal(size=(9, 9)) * 5)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    assert not np.triu(P, 1).any()
    assert P[0, 0] == 1.0


def test_equal_scores_average_the_prefix():
    # K = 0: every causal score is 0, so row i averages V_0..V_i
    rng = np.random.default_rng(3)
    n, heads, dh = 7, 2, 3
    Q, V = rng.normal(size=(n, heads * dh)), rng.normal(size=(n, heads * dh))
    ctx = TR.attention(Q, np.zeros_like(Q), V, heads)
    np.testing.assert_allclose(ctx, np.cumsum(V, axis=0) / np.arange(1, n + 1)[:, None],
                               rtol=0, atol=1e-14)


def test_single_token_takes_its_own_value():
    rng = np.random.default_rng(4)
    d, heads = 8, 2
    w = _weights(rng, d, heads, 16)
    X = rng.normal(size=(1, d))
    _, it = TR.user_fwd(X, w, heads, 1e-6, return_intermediates=True)
    np.testing.assert_allclose(it["ctx"], it["QKV"][:, 2 * d:], rtol=0, atol=1e-14)


def test_causal_and_users_independent():
    rng = np.random.default_rng(5)
    d, heads = 8, 2
    w = _weights(rng, d, heads, 16)
    X = rng.normal(size=(12, d))
    off = np.array([0, 5, 12])
    Y = TR.layer_fwd(X, off, w, heads, 1e-6)
    X2 = X.copy()
    X2[3] += 10.0                       # a later token of user 0
    X2[8] -= 4.0                        # user 1
    Y2 = TR.layer_fwd(X2, off, w, heads, 1e-6)
    np.testing.assert_array_equal(Y2[:3], Y[:3])
    assert not np.allclose(Y2[3:5], Y[3:5])
    np.testing.assert_array_equal(Y2[5:8], Y[5:8])


def test_planted_mistakes_are_caught():
    rng = np.random.default_rng(6)
    n, heads, dh = 10, 2, 4
    Q, K, V = (rng.normal(size=(n, heads * dh)) for _ in range(3))
    good = TR.attention(Q, K, V, heads)
    # no 1/sqrt(d_h) scale
    bad = TR.attention(Q * math.sqrt(dh), K, V, heads)
    assert np.abs(bad - good).max() > 1e-3
    # non-causal softmax
    S = Q[:, :dh] @ K[:, :dh].T / math.sqrt(dh)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    full = (E / E.sum(axis=1, keepdims=True)) @ V[:, :dh]
    assert np.abs(full - good[:, :dh]).max() > 1e-3
    # Q and K swapped
    assert np.abs(TR.attention(K, Q, V, heads) - good).max() > 1e-3


def test_rows_helper_equals_the_whole_user():
    rng = np.random.default_rng(7)
    d, heads = 8, 2
    w = _weights(rng, d, heads, 16)
    X = rng.normal(size=(20, d))
    rows = [0, 3, 19, 7]
    np.testing.assert_allclose(TR.user_rows(X, w, heads, 1e-6, rows),
                               TR.user_fwd(X, w, heads, 1e-6)[rows], rtol=0, atol=1e-12)
