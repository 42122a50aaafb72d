"""Float64 CPU oracle for the HSTU layer stack and M-FALCON ranking.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA path never
calls it, and it shares no code with the CUDA path.

Source of every definition: the page 'HSTUとGenerative Recommenders――行動履歴から
1.5兆parameterの推薦モデルへ' (koktn.github.io, an explainer of Zhai et al.,
ICML 2024), section 'HSTUはTransformerと何が違うのか' and its subsections, and
section '長い履歴を現実の計算量へ収める4つの工夫' (M-FALCON).  Where the page is
silent the readings are stated next to the code (bucket function, 1/n
normaliser, split order, biases, epsilon, candidate position/time).

Per user b with rows i, j in 0..n_b-1, one layer computes

  1. G = SiLU(X W1^T + b1), split column-wise into [U | V | Q | K]
     (subsection '1. U、V、Q、Kは同じ入力を見る4つの役割': one projection f1,
     SiLU, split into four roles; Q,K are h x N x d_qk, U,V are h x N x d_v).
  2. s_ij = Q_i . K_j + pos_bias(i - j) + time_bias(t_i - t_j) for j <= i
     (subsection '2. QKᵀで「どの履歴を見るか」を決める': score equation, causal).
  3. O_i = (1/n_b) sum_{j<=i} SiLU(s_ij) V_j   (same subsection: pointwise
     SiLU weights, no softmax; the 1/n_b normaliser is the reading of
     "normalised by sequence length").
  4. Z_i = LayerNorm(O_i) * U_i  (subsection '3. Uでcontextをgateし、次のlayerへ渡す').
  5. Y_i = X_i + Z_i W2^T + b2   (same subsection: f2 back to d, residual).

Every pin of this file lives in ``tests/test_oracle_pins.py``; no function
here is "parity unpinned".
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "log_bucket", "silu", "layer_norm", "split_uvqk", "layer_fwd", "stack_fwd",
    "layer_rows", "stack_user", "mfalcon_rank", "mfalcon_user",
]


# ---------------------------------------------------------------------------
# elementary functions
# ---------------------------------------------------------------------------
def log_bucket(x, n_buckets: int, sub_bits: int) -> np.ndarray:
    """Log-linear bucket of a non-negative integer distance.

    The page says only that the relative bias is indexed by sequence distance
    and by elapsed real time; the bucket rule is a reading made here: values
    below 2^S keep their own bucket; above, with e = floor(log2 x), the bucket
    is (e - S + 1) * 2^S + ((x >> (e - S)) - 2^S), i.e. the exponent and the
    top S mantissa bits of x; clamped to n_buckets - 1.
    """
    x = np.asarray(x, dtype=np.int64)
    if x.size and int(x.min()) < 0:
        raise ValueError("log_bucket takes non-negative distances")
    if x.size and int(x.max()) >= (1 << 53):
        raise ValueError("distances beyond 2^53 are outside the oracle's exact range")
    S = int(sub_bits)
    out = x.copy()
    big = x >= (1 << S)
    if np.any(big):
        xb = x[big]
        # frexp is exact for integers below 2^53: x = m * 2^p, m in [0.5, 1)
        _, p = np.frexp(xb.astype(np.float64))
        e = p.astype(np.int64) - 1
        out[big] = (e - S + 1) * (1 << S) + ((xb >> (e - S)) - (1 << S))
    return np.minimum(out, n_buckets - 1)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x / (1 + exp(-x))."""
    x = np.asarray(x, dtype=np.float64)
    # split by sign so exp never overflows
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = x[pos] / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = x[~pos] * ex / (1.0 + ex)
    return out


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis (biased variance), then gamma, beta."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def split_uvqk(G: np.ndarray, dims) -> Dict[str, np.ndarray]:
    """Split f1's output column-wise in the order U, V, Q, K (head-major inside
    each part)."""
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    a, b, c = h * dv, 2 * h * dv, 2 * h * dv + h * dqk
    return dict(U=G[:, :a], V=G[:, a:b], Q=G[:, b:c], K=G[:, c:c + h * dqk])


def _w64(w: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    return {k: np.asarray(v, dtype=np.float64) for k, v in w.items()}


# ---------------------------------------------------------------------------
# one user, one layer (dense over that user's rows)
# ---------------------------------------------------------------------------
def _attention_user(Q, K, V, t, w, dims, norm: float, rows: Optional[np.ndarray] = None):
    """O rows for one user: causal pointwise attention with the relative bias.

    Q, K, V: that user's rows (all n); t: int64 timestamps; rows: the query
    rows to compute (default all).  Returns [len(rows), h*dv].
    """
    n = Q.shape[0]
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    if rows is None:
        rows = np.arange(n)
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), h * dv))
    if n == 0 or len(rows) == 0:
        return out
    j = np.arange(n)
    dist = rows[:, None] - j[None, :]                      # i - j
    causal = dist >= 0
    pb = log_bucket(np.where(causal, dist, 0), dims.n_pos_buckets, dims.pos_sub_bits)
    gap = np.maximum(t[rows][:, None] - t[None, :], 0)
    tb = log_bucket(gap, dims.n_time_buckets, dims.time_sub_bits)
    for k in range(h):
        qk = Q[rows, k * dqk:(k + 1) * dqk] @ K[:, k * dqk:(k + 1) * dqk].T
        s = qk + w["rab_pos"][k][pb] + w["rab_time"][k][tb]
        A = np.where(causal, silu(s), 0.0)
        out[:, k * dv:(k + 1) * dv] = (A @ V[:, k * dv:(k + 1) * dv]) / norm
    return out


def layer_fwd(X, offsets, timestamps, w, dims, norm_len: Optional[Sequence[int]] = None,
              return_intermediates: bool = False):
    """One HSTU layer over a jagged batch.  X: [T, d]; offsets: int64 [B+1].

    ``norm_len`` overrides the per-user normaliser (default: the user's own
    length n_b; an empty user has nothing to normalise).  With
    ``return_intermediates`` also returns U, V, Q, K, O (pre-LayerNorm) and Z.
    """
    X = np.asarray(X, dtype=np.float64)
    w = _w64(w)
    offsets = np.asarray(offsets, dtype=np.int64)
    t_all = np.asarray(timestamps, dtype=np.int64)
    G = silu(X @ w["W1"].T + w["b1"])
    parts = split_uvqk(G, dims)
    T = X.shape[0]
    O = np.zeros((T, dims.n_heads * dims.d_v))
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        if n == 0:
            continue
        norm = float(n if norm_len is None else norm_len[b])
        O[s:e] = _attention_user(parts["Q"][s:e], parts["K"][s:e], parts["V"][s:e],
                                 t_all[s:e], w, dims, norm)
    Z = layer_norm(O, w["ln_gamma"], w["ln_beta"], dims.ln_eps) * parts["U"]
    Y = X + Z @ w["W2"].T + w["b2"]
    if return_intermediates:
        return Y, dict(G=G, O=O, Z=Z, **parts)
    return Y


def stack_fwd(X, offsets, timestamps, weights: List[Dict[str, np.ndarray]], dims,
              norm_len=None):
    """L layers, each layer's output feeding the next (residual stacking)."""
    Y = np.asarray(X, dtype=np.float64)
    for w in weights:
        Y = layer_fwd(Y, offsets, timestamps, w, dims, norm_len=norm_len)
    return Y


def layer_rows(X_user, t_user, w, dims, rows):
    """Layer outputs for selected rows of ONE user (rows depend only on
    earlier rows of the same user, so only those rows' outputs are formed).
    X_user: [n, d] that user's rows.  Returns ([len(rows), d], intermediates)."""
    X_user = np.asarray(X_user, dtype=np.float64)
    w = _w64(w)
    rows = np.asarray(rows, dtype=np.int64)
    n = X_user.shape[0]
    G = silu(X_user @ w["W1"].T + w["b1"])
    parts = split_uvqk(G, dims)
    O = _attention_user(parts["Q"], parts["K"], parts["V"], np.asarray(t_user, np.int64),
                        w, dims, float(n), rows)
    Z = layer_norm(O, w["ln_gamma"], w["ln_beta"], dims.ln_eps) * parts["U"][rows]
    Y = X_user[rows] + Z @ w["W2"].T + w["b2"]
    return Y, dict(O=O, Z=Z, U=parts["U"][rows], V=parts["V"][rows],
                   Q=parts["Q"][rows], K=parts["K"][rows])


def stack_user(X_user, t_user, weights, dims):
    """All L layers for one user (all rows)."""
    n = X_user.shape[0]
    off = np.array([0, n], dtype=np.int64)
    return stack_fwd(X_user, off, t_user, weights, dims)


# ---------------------------------------------------------------------------
# M-FALCON
# ---------------------------------------------------------------------------
def mfalcon_user(hist_X, hist_t, cand_X, t_req, microbatch: int, head_vec, weights, dims):
    """Scores of one user's candidates.

    Section '4. M-FALCONで候補間の履歴計算を共有する': candidates are grouped in
    microbatches of size b_m and appended after the history; the attention
    mask and relative bias are adjusted so that each candidate sees the whole
    history and itself but no other candidate, and the history's per-layer
    K/V is computed once and reused by every microbatch.

    Readings: every candidate sits at position n (distance n - j to history
    row j, 0 to itself) and at time t_req (gap max(0, t_req - t_j)); its
    normaliser is the history length n (so the history rows' outputs, and so
    the cached K/V, do not depend on the candidates).  The score is the dot
    of the last layer's candidate output with the head vector.
    """
    hist_X = np.asarray(hist_X, dtype=np.float64)
    cand_X = np.asarray(cand_X, dtype=np.float64)
    hist_t = np.asarray(hist_t, dtype=np.int64)
    n = hist_X.shape[0]
    m = cand_X.shape[0]
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    norm = float(max(n, 1))
    # history pass: per-layer K, V cache (history rows never see candidates)
    cache = []
    Xh = hist_X
    off = np.array([0, n], dtype=np.int64)
    for w in weights:
        Yh, inter = layer_fwd(Xh, off, hist_t, w, dims, return_intermediates=True)
        cache.append((inter["K"], inter["V"]))
        Xh = Yh
    # relative bias of a candidate towards history row j (same for every candidate)
    j = np.arange(n)
    pb_hist = log_bucket(n - j, dims.n_pos_buckets, dims.pos_sub_bits)
    tb_hist = log_bucket(np.maximum(t_req - hist_t, 0), dims.n_time_buckets, dims.time_sub_bits)
    pb_self = log_bucket(np.zeros(1, np.int64), dims.n_pos_buckets, dims.pos_sub_bits)[0]
    tb_self = log_bucket(np.zeros(1, np.int64), dims.n_time_buckets, dims.time_sub_bits)[0]
    scores = np.zeros(m)
    bm = max(1, int(microbatch))
    for c0 in range(0, m, bm):
        Xc = cand_X[c0:c0 + bm]
        mb = Xc.shape[0]
        # appended block: columns = [history (n) | this microbatch (mb)]
        vis = np.concatenate([np.ones((mb, n), bool), np.eye(mb, dtype=bool)], axis=1)
        for (Kh, Vh), w in zip(cache, weights):
            w = _w64(w)
            Gc = silu(Xc @ w["W1"].T + w["b1"])
            pc = split_uvqk(Gc, dims)
            Oc = np.zeros((mb, h * dv))
            for k in range(h):
                qs, vs = slice(k * dqk, (k + 1) * dqk), slice(k * dv, (k + 1) * dv)
                keys = np.concatenate([Kh[:, qs], pc["K"][:, qs]], axis=0)
                vals = np.concatenate([Vh[:, vs], pc["V"][:, vs]], axis=0)
                bias = np.concatenate([
                    np.broadcast_to(w["rab_pos"][k][pb_hist] + w["rab_time"][k][tb_hist], (mb, n)),
                    np.full((mb, mb), w["rab_pos"][k][pb_self] + w["rab_time"][k][tb_self]),
                ], axis=1)
                s = pc["Q"][:, qs] @ keys.T + bias
                A = np.where(vis, silu(s), 0.0)
                Oc[:, vs] = (A @ vals) / norm
            Zc = layer_norm(Oc, w["ln_gamma"], w["ln_beta"], dims.ln_eps) * pc["U"]
            Xc = Xc + Zc @ w["W2"].T + w["b2"]
        scores[c0:c0 + mb] = Xc @ np.asarray(head_vec, np.float64)
    return scores


def mfalcon_rank(hist_X, hist_offsets, hist_t, cand_X, cand_offsets, request_ts, microbatch,
                 head_vec, weights, dims, users: Optional[Sequence[int]] = None):
    """Scores for every candidate (or only those of ``users``), float64 [C]."""
    hist_offsets = np.asarray(hist_offsets, np.int64)
    cand_offsets = np.asarray(cand_offsets, np.int64)
    B = len(hist_offsets) - 1
    out = np.full(int(cand_offsets[-1]), np.nan)
    for b in (range(B) if users is None else users):
        hs, he = int(hist_offsets[b]), int(hist_offsets[b + 1])
        cs, ce = int(cand_offsets[b]), int(cand_offsets[b + 1])
        if ce == cs:
            continue
        t_req = int(request_ts[b]) if request_ts is not None else (int(hist_t[he - 1]) if he > hs else 0)
        out[cs:ce] = mfalcon_user(hist_X[hs:he], hist_t[hs:he], cand_X[cs:ce], t_req,
                                  microbatch, head_vec, weights, dims)
    return out
