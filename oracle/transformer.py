"""Oracle for the softmax-Transformer encoder layer used as the comparator of
the HSTU layer (test infrastructure only: the GPU path never imports this
module).

Sources:
* The GenRec explainer on techistory.net (scratchpad page 13), the attention
  equations and the toy SimpleSelfAttention: Q = X W_Q, K = X W_K, V = X W_V
  without biases, per head softmax(Q K^T / sqrt(d_k)) V, the heads
  concatenated and projected by W_O.
* 'HSTUとGenerative Recommenders', section '2. QKᵀで「どの履歴を見るか」を決める'
  (an ordinary Transformer normalises each query's scores with a softmax so
  that the weights over the history sum to 1; HSTU applies SiLU instead), and
  section 'Production評価の12.4%をどう読むか' (the efficiency comparison against
  a FlashAttention-2 Transformer at 8,192 tokens, d = 512, 8 heads).

Read as a standard pre-LayerNorm encoder layer over each user's sequence,
causal like the HSTU layer it is compared with:
    A  = LN1(X)
    Q, K, V = A W_Q^T, A W_K^T, A W_V^T          (W_QKV = [W_Q; W_K; W_V])
    ctx_h = softmax_causal(Q_h K_h^T / sqrt(d_h)) V_h
    X1 = X + ctx W_O^T
    Y  = X1 + SiLU(LN2(X1) W_1^T + b_1) W_2^T + b_2
(the feed-forward activation is SiLU; LayerNorm with gamma, beta and eps).
Plain numpy float64, one user at a time.
"""
from __future__ import annotations

import math
from typing import Dict

import numpy as np


def layer_norm(x, gamma, beta, eps):
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def silu(x):
    return x / (1.0 + np.exp(-x))


def softmax_causal(S):
    """Row-wise softmax of S [n, n] over columns j <= i."""
    n = S.shape[0]
    S = np.where(np.tril(np.ones((n, n), bool)), S, -np.inf)
    S = S - S.max(axis=1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=1, keepdims=True)


def attention(Q, K, V, n_heads: int):
    """Causal multi-head softmax attention of one user: ctx [n, h*d_h]."""
    n = Q.shape[0]
    dh = Q.shape[1] // n_heads
    out = np.empty((n, n_heads * dh))
    for h in range(n_heads):
        q, k, v = (M[:, h * dh:(h + 1) * dh] for M in (Q, K, V))
        P = softmax_causal(q @ k.T / math.sqrt(dh))
        out[:, h * dh:(h + 1) * dh] = P @ v
    return out


def user_fwd(X, w: Dict[str, np.ndarray], n_heads: int, eps: float, return_intermediates=False):
    X = np.asarray(X, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in w.items()}
    d = X.shape[1]
    A = layer_norm(X, W["ln1_gamma"], W["ln1_beta"], eps)
    QKV = A @ W["W_qkv"].T
    Q, K, V = QKV[:, :d], QKV[:, d:2 * d], QKV[:, 2 * d:]
    ctx = attention(Q, K, V, n_heads)
    X1 = X + ctx @ W["W_o"].T
    B = layer_norm(X1, W["ln2_gamma"], W["ln2_beta"], eps)
    F = silu(B @ W["W_1"].T + W["b_1"])
    Y = X1 + F @ W["W_2"].T + W["b_2"]
    if return_intermediates:
        return Y, dict(A=A, QKV=QKV, ctx=ctx, X1=X1, B=B, F=F)
    return Y


def layer_fwd(X, offsets, w, n_heads: int, eps: float):
    """The layer over a jagged batch (users independent)."""
    X = np.asarray(X, np.float64)
    Y = np.empty_like(X)
    offsets = np.asarray(offsets, np.int64)
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e > s:
            Y[s:e] = user_fwd(X[s:e], w, n_heads, eps)
    return Y


def user_rows(X, w, n_heads: int, eps: float, rows):
    """Y at the given rows of one user only (the keys and values of every row
    up to the last requested one are formed; the rest of the layer runs on the
    requested rows).  Equal to user_fwd(X, ...)[rows]."""
    X = np.asarray(X, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in w.items()}
    rows = np.asarray(rows, np.int64)
    d = X.shape[1]
    dh = d // n_heads
    last = int(rows.max()) + 1
    A = layer_norm(X[:last], W["ln1_gamma"], W["ln1_beta"], eps)
    QKV = A @ W["W_qkv"].T
    ctx = np.empty((len(rows), d))
    for ri, i in enumerate(rows):
        for h in range(n_heads):
            q = QKV[i, h * dh:(h + 1) * dh]
            k = QKV[:i + 1, d + h * dh:d + (h + 1) * dh]
            v = QKV[:i + 1, 2 * d + h * dh:2 * d + (h + 1) * dh]
            s = k @ q / math.sqrt(dh)
            p = np.exp(s - s.max())
            ctx[ri, h * dh:(h + 1) * dh] = (p / p.sum()) @ v
    X1 = X[rows] + ctx @ W["W_o"].T
    B = layer_norm(X1, W["ln2_gamma"], W["ln2_beta"], eps)
    F = silu(B @ W["W_1"].T + W["b_1"])
    return X1 + F @ W["W_2"].T + W["b_2"]
