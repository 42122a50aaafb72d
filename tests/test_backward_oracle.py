"""Pins of the HSTU layer's backward oracle (oracle.hstu_backward): central
finite differences of the forward oracle, and torch autograd through an
independently written torch forward, on a tiny jagged batch (empty, length-1
and longer users)."""
import numpy as np
import torch

import hstu_workloads as hw
from oracle import hstu_oracle as F
from oracle import hstu_backward as BW

DIMS = hw.LayerDims(8, 2, 4, 4, 8, 8, 1, 1, 1e-6, hw.FP32)
LENGTHS = [3, 0, 1, 5]


def _case(seed=0):
    rng = np.random.default_rng(seed)
    d, F_ = DIMS.d_model, DIMS.f1_width
    w = dict(W1=rng.normal(0, 0.5, (F_, d)), b1=rng.normal(0, 0.2, F_),
             W2=rng.normal(0, 0.5, (d, DIMS.hdv)), b2=rng.normal(0, 0.2, d),
             ln_gamma=1 + rng.normal(0, 0.2, DIMS.hdv), ln_beta=rng.normal(0, 0.2, DIMS.hdv),
             rab_pos=rng.normal(0, 0.3, (DIMS.n_heads, DIMS.n_pos_buckets)),
             rab_time=rng.normal(0, 0.3, (DIMS.n_heads, DIMS.n_time_buckets)))
    off = np.concatenate([[0], np.cumsum(LENGTHS)]).astype(np.int64)
    T = int(off[-1])
    X = rng.normal(size=(T, d))
    ts = np.concatenate([np.sort(rng.integers(0, 50, n)) for n in LENGTHS]).astype(np.int64)
    dY = rng.normal(size=(T, d))
    return X, off, ts, w, dY


def _objective(X, off, ts, w, dY):
    return float((dY * F.layer_fwd(X, off, ts, w, DIMS)).sum())


def test_matches_central_finite_differences():
    X, off, ts, w, dY = _case(0)
    g = BW.layer_bwd(X, off, ts, w, DIMS, dY)
    eps = 1e-6
    for name in ["dX"] + ["d" + k for k in w]:
        key = name[1:]
        base = X if key == "X" else w[key]
        got = g[name]
        num = np.empty_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            if key == "X":
                fp = _objective(plus, off, ts, w, dY)
                fm = _objective(minus, off, ts, w, dY)
            else:
                fp = _objective(X, off, ts, {**w, key: plus}, dY)
                fm = _objective(X, off, ts, {**w, key: minus}, dY)
            num[idx] = (fp - fm) / (2 * eps)
        scale = max(1.0, float(np.abs(num).max()))
        assert np.abs(got - num).max() <= 1e-6 * scale, (name, np.abs(got - num).max())


def _torch_forward(X, off, ts, w):
    """The layer in torch float64, written independently of the oracle."""
    h, dqk, dv = DIMS.n_heads, DIMS.d_qk, DIMS.d_v
    G = torch.nn.functional.silu(X @ w["W1"].T + w["b1"])
    U, V = G[:, :h * dv], G[:, h * dv:2 * h * dv]
    Q = G[:, 2 * h * dv:2 * h * dv + h * dqk]
    K = G[:, 2 * h * dv + h * dqk:]
    outs = []
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        n = e - s
        if n == 0:
            continue
        i = np.arange(n)
        dist = i[:, None] - i[None, :]
        pb = torch.from_numpy(F.log_bucket(np.maximum(dist, 0), DIMS.n_pos_buckets,
                                           DIMS.pos_sub_bits))
        gap = np.maximum(ts[s:e][:, None] - ts[s:e][None, :], 0)
        tb = torch.from_numpy(F.log_bucket(gap, DIMS.n_time_buckets, DIMS.time_sub_bits))
        mask = torch.from_numpy(dist >= 0)
        heads = []
        for k in range(h):
            S = (Q[s:e, k * dqk:(k + 1) * dqk] @ K[s:e, k * dqk:(k + 1) * dqk].T
                 + w["rab_pos"][k][pb] + w["rab_time"][k][tb])
            A = torch.where(mask, torch.nn.functional.silu(S), torch.zeros_like(S))
            heads.append(A @ V[s:e, k * dv:(k + 1) * dv] / n)
        outs.append(torch.cat(heads, dim=1))
    O = torch.cat(outs, dim=0)
    Ln = torch.nn.functional.layer_norm(O, (h * dv,), w["ln_gamma"], w["ln_beta"], DIMS.ln_eps)
    return X + (Ln * U) @ w["W2"].T + w["b2"]


def test_matches_torch_autograd():
    X, off, ts, w, dY = _case(1)
    g = BW.layer_bwd(X, off, ts, w, DIMS, dY)
    tX = torch.tensor(X, requires_grad=True)
    tw = {k: torch.tensor(v, requires_grad=True) for k, v in w.items()}
    Y = _torch_forward(tX, off, ts, tw)
    np.testing.assert_allclose(Y.detach().numpy(), F.layer_fwd(X, off, ts, w, DIMS), atol=1e-12)
    (Y * torch.from_numpy(dY)).sum().backward()
    np.testing.assert_allclose(g["dX"], tX.grad.numpy(), rtol=0, atol=1e-10)
    for k, v in tw.items():
        np.testing.assert_allclose(g["d" + k], v.grad.numpy(), rtol=0, atol=1e-10, err_msg=k)


def test_silu_derivative_closed_form():
    x = np.array([-30.0, -2.0, -0.5, 0.0, 0.5, 2.0, 30.0])
    sig = 1 / (1 + np.exp(-x))
    np.testing.assert_allclose(BW.silu_grad(x), sig + x * sig * (1 - sig), rtol=1e-14, atol=1e-14)
    assert BW.silu_grad(np.array([0.0]))[0] == 0.5


def test_stack_matches_finite_differences():
    X, off, ts, w0, dY = _case(2)
    w1 = {k: v * 0.9 + 0.01 for k, v in _case(3)[3].items()}
    ws = [w0, w1]
    dX, gs = BW.stack_bwd(X, off, ts, ws, DIMS, dY)

    def obj(Xv, wl):
        return float((dY * F.stack_fwd(Xv, off, ts, wl, DIMS)).sum())
    eps = 1e-6
    rng = np.random.default_rng(4)
    # every input entry, and a random subset of each layer's parameters
    num = np.empty_like(X)
    for idx in np.ndindex(X.shape):
        p, m = X.copy(), X.copy()
        p[idx] += eps
        m[idx] -= eps
        num[idx] = (obj(p, ws) - obj(m, ws)) / (2 * eps)
    assert np.abs(dX - num).max() <= 1e-6 * max(1.0, np.abs(num).max())
    for layer in range(2):
        for key, val in ws[layer].items():
            for _ in range(3):
                idx = tuple(int(rng.integers(0, n)) for n in val.shape)
                p = [dict(wl) for wl in ws]
                m = [dict(wl) for wl in ws]
                p[layer][key] = val.copy()
                m[layer][key] = val.copy()
                p[layer][key][idx] += eps
                m[layer][key][idx] -= eps
                fd = (obj(X, p) - obj(X, m)) / (2 * eps)
                got = gs[layer]["d" + key][idx]
                assert abs(got - fd) <= 1e-6 * max(1.0, abs(fd)), (layer, key, idx, got, fd)
