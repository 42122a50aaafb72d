"""Float64 CPU oracle of the gradients of the HSTU layer and stack (the backward pass,
for training).  TEST INFRASTRUCTURE ONLY: only ``tests/`` may import it; no
kernel of the library computes a backward pass yet.

Source: the forward pass of 'HSTUとGenerative Recommenders', section
'HSTUはTransformerと何が違うのか' and its subsections (the same definitions as
``oracle.hstu_oracle``, whose forward functions this module calls), and
section 'Production評価の12.4%をどう読むか' (training is where the pages report
the largest gain over a FlashAttention-2 Transformer).  The gradients are the
derivatives of that forward written out by the chain rule, step by step in
reverse order; for user b (rows i, j of that user, n = n_b) and head k:

  Y = X + Z W2^T + b2           dW2 = dY^T Z, db2 = sum dY, dZ = dY W2, dX = dY
  Z = L * U,  L = LN(O)g + be    dL = dZ * U, dU = dZ * L
  L = xhat g + be               dg = sum dL xhat, dbe = sum dL,
                                dO = (dxh - mean(dxh) - xhat mean(dxh xhat)) / sd,
                                dxh = dL g   (per row, over the h*d_v features)
  O_i = (1/n) sum_{j<=i} A_ij V_j      dA = (1/n) dO V^T (j <= i), dV = (1/n) A^T dO
  A = SiLU(S)                   dS = dA SiLU'(S),
                                SiLU'(s) = sig(s) (1 + s (1 - sig(s)))
  S = Q K^T + rp[pb(i-j)] + rt[tb(t_i-t_j)]
                                dQ = dS K, dK = dS^T Q,
                                drp[k][b] = sum over (i,j) in bucket b of dS,
                                drt likewise over the time buckets
  G = SiLU(P), P = X W1^T + b1   dP = [dU|dV|dQ|dK] SiLU'(P),
                                dW1 = dP^T X, db1 = sum dP, dX += dP W1.
Plain numpy, one user at a time.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from oracle import hstu_oracle as F


def _sigmoid(x):
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    e = np.exp(x[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def silu_grad(x):
    """d SiLU(x) / dx = sig(x) (1 + x (1 - sig(x)))."""
    s = _sigmoid(x)
    return s * (1.0 + np.asarray(x, np.float64) * (1.0 - s))


def layer_bwd(X, offsets, timestamps, w: Dict[str, np.ndarray], dims, dY):
    """Gradients of sum(dY * Y) for Y = layer_fwd(X, ...): returns a dict with
    dX and one entry per weight (dW1, db1, dW2, db2, dln_gamma, dln_beta,
    drab_pos, drab_time)."""
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in w.items()}
    off = np.asarray(offsets, np.int64)
    t_all = np.asarray(timestamps, np.int64)
    h, dqk, dv, eps = dims.n_heads, dims.d_qk, dims.d_v, dims.ln_eps
    hdv = h * dv
    # forward intermediates
    P = X @ W["W1"].T + W["b1"]
    G = F.silu(P)
    parts = F.split_uvqk(G, dims)
    U, V, Q, K = parts["U"], parts["V"], parts["Q"], parts["K"]
    _, it = F.layer_fwd(X, off, t_all, w, dims, return_intermediates=True)
    O = it["O"]
    mu = O.mean(axis=1, keepdims=True)
    sd = np.sqrt(((O - mu) ** 2).mean(axis=1, keepdims=True) + eps)
    xhat = (O - mu) / sd
    L = xhat * W["ln_gamma"] + W["ln_beta"]
    Z = L * U
    g = {}
    # Y = X + Z W2^T + b2
    g["dW2"] = dY.T @ Z
    g["db2"] = dY.sum(axis=0)
    dZ = dY @ W["W2"]
    dX = dY.copy()
    # Z = L * U
    dL = dZ * U
    dU = dZ * L
    # LayerNorm
    g["dln_gamma"] = (dL * xhat).sum(axis=0)
    g["dln_beta"] = dL.sum(axis=0)
    dxh = dL * W["ln_gamma"]
    dO = (dxh - dxh.mean(axis=1, keepdims=True)
          - xhat * (dxh * xhat).mean(axis=1, keepdims=True)) / sd
    # attention, per user and head
    dV = np.zeros_like(V)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    drp = np.zeros_like(W["rab_pos"])
    drt = np.zeros_like(W["rab_time"])
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        n = e - s
        if n == 0:
            continue
        i = np.arange(n)
        dist = i[:, None] - i[None, :]
        causal = dist >= 0
        pb = F.log_bucket(np.where(causal, dist, 0), dims.n_pos_buckets, dims.pos_sub_bits)
        t = t_all[s:e]
        tb = F.log_bucket(np.maximum(t[:, None] - t[None, :], 0), dims.n_time_buckets,
                          dims.time_sub_bits)
        for k in range(h):
            qs, vs = slice(k * dqk, (k + 1) * dqk), slice(k * dv, (k + 1) * dv)
            Qk, Kk, Vk = Q[s:e, qs], K[s:e, qs], V[s:e, vs]
            S = Qk @ Kk.T + W["rab_pos"][k][pb] + W["rab_time"][k][tb]
            A = np.where(causal, F.silu(S), 0.0)
            dOk = dO[s:e, vs]
            dA = np.where(causal, dOk @ Vk.T / n, 0.0)
            dV[s:e, vs] += A.T @ dOk / n
            dS = np.where(causal, dA * silu_grad(S), 0.0)
            dQ[s:e, qs] += dS @ Kk
            dK[s:e, qs] += dS.T @ Qk
            np.add.at(drp[k], pb[causal], dS[causal])
            np.add.at(drt[k], tb[causal], dS[causal])
    g["drab_pos"], g["drab_time"] = drp, drt
    # G = SiLU(P), split [U | V | Q | K]
    dG = np.concatenate([dU, dV, dQ, dK], axis=1)
    dP = dG * silu_grad(P)
    g["dW1"] = dP.T @ X
    g["db1"] = dP.sum(axis=0)
    dX += dP @ W["W1"]
    g["dX"] = dX
    return g


def stack_bwd(X, offsets, timestamps, weights, dims, dY):
    """Gradients of sum(dY * Y) for Y = stack_fwd(X, ...) (layers applied in
    order, each output the next layer's input): the layers' backward passes
    in reverse order, each fed the gradient of its own output and its own
    input.  Returns (dX, [per-layer weight gradients])."""
    inputs = [np.asarray(X, np.float64)]
    for w in weights[:-1]:
        inputs.append(F.layer_fwd(inputs[-1], offsets, timestamps, w, dims))
    grads = [None] * len(weights)
    g_out = np.asarray(dY, np.float64)
    for layer in range(len(weights) - 1, -1, -1):
        g = layer_bwd(inputs[layer], offsets, timestamps, weights[layer], dims, g_out)
        g_out = g.pop("dX")
        grads[layer] = g
    return g_out, grads
