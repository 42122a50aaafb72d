"""Float64 emulation of the backward kernels' fp16 rounding points, applied to
the oracle's arithmetic (test infrastructure, run by hand: python
tests/bwd_rounding_emulation.py).  It reproduces the error figures quoted in
tests/test_gpu_backward.py: which rounding point dominates the error of dX
and of the bottom layer's dW1 in the two-layer stack test, and that the
dominant part comes from one user of one token (a row whose LayerNorm
amplifies the rounding of the f1 output).  Rounding points: 'pre' / 'G' the
f1 pre-activation and output, 'xn' the normalised O, 'gyh' the fp16 copy of
the output gradient, 'Z', 'dO', 'P' and 'dS' in attention, 'dP' the f1
gradient, 'fwdP' the forward's P.
"""
import os, sys
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import numpy as np, hstu_workloads as hw
from oracle import hstu_oracle as F
from oracle import hstu_backward as BW
from gpu_util import relerr, rmserr

def f16(a): return np.asarray(a, np.float64).astype(np.float16).astype(np.float64)

def layer_bwd_emu(X, off, ts, w, dims, dY, R):
    # R: set of rounding points to apply
    X = np.asarray(X, np.float64); dY = np.asarray(dY, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in w.items()}
    h, dqk, dv, eps = dims.n_heads, dims.d_qk, dims.d_v, dims.ln_eps
    P = X @ W["W1"].T + W["b1"]
    if 'pre' in R: Pq = f16(P)
    else: Pq = P
    G = F.silu(P)
    if 'G' in R: G = f16(G)
    parts = F.split_uvqk(G, dims)
    U, V, Q, K = parts["U"], parts["V"], parts["Q"], parts["K"]
    T = X.shape[0]
    O = np.zeros((T, h*dv))
    for b in range(len(off)-1):
        s, e = int(off[b]), int(off[b+1]); n = e - s
        if n == 0: continue
        if 'fwdP' in R:
            i = np.arange(n); dist = i[:, None]-i[None, :]; causal = dist >= 0
            pb = F.log_bucket(np.where(causal, dist, 0), dims.n_pos_buckets, dims.pos_sub_bits)
            t = ts[s:e]; tb = F.log_bucket(np.maximum(t[:, None]-t[None, :], 0), dims.n_time_buckets, dims.time_sub_bits)
            for k in range(h):
                qs, vs = slice(k*dqk, (k+1)*dqk), slice(k*dv, (k+1)*dv)
                S = Q[s:e, qs]@K[s:e, qs].T + W["rab_pos"][k][pb] + W["rab_time"][k][tb]
                A = np.where(causal, f16(F.silu(S)), 0.0)
                O[s:e, vs] = A@V[s:e, vs]/n
        else:
            O[s:e] = F._attention_user(Q[s:e], K[s:e], V[s:e], ts[s:e], W, dims, float(n))
    if 'xn' in R:
        Oh = O.reshape(T, h, dv); m = Oh.mean(2, keepdims=True); sd = np.sqrt(((Oh-m)**2).mean(2, keepdims=True))
        xn = np.where(sd > 0, (Oh - m)/np.where(sd>0, sd, 1), 0); O = (m + sd * f16(xn)).reshape(T, h*dv)
    mu = O.mean(1, keepdims=True); sd = np.sqrt(((O-mu)**2).mean(1, keepdims=True) + eps)
    xhat = (O - mu)/sd; L = xhat*W["ln_gamma"] + W["ln_beta"]; Z = L*U
    dYh = f16(dY) if 'gyh' in R else dY
    g = {}
    Zq = f16(Z) if 'Z' in R else Z
    g["dW2"] = dYh.T @ Zq; g["db2"] = dY.sum(0)
    dZ = dYh @ W["W2"]
    dX = dY.copy()
    dL = dZ*U; dU = dZ*L
    g["dln_gamma"] = (dL*xhat).sum(0); g["dln_beta"] = dL.sum(0)
    dxh = dL*W["ln_gamma"]
    dO = (dxh - dxh.mean(1, keepdims=True) - xhat*(dxh*xhat).mean(1, keepdims=True))/sd
    if 'dO' in R: dO = f16(dO)
    dV = np.zeros_like(V); dQ = np.zeros_like(Q); dK = np.zeros_like(K)
    for b in range(len(off)-1):
        s, e = int(off[b]), int(off[b+1]); n = e - s
        if n == 0: continue
        i = np.arange(n); dist = i[:, None]-i[None, :]; causal = dist >= 0
        pb = F.log_bucket(np.where(causal, dist, 0), dims.n_pos_buckets, dims.pos_sub_bits)
        t = ts[s:e]; tb = F.log_bucket(np.maximum(t[:, None]-t[None, :], 0), dims.n_time_buckets, dims.time_sub_bits)
        for k in range(h):
            qs, vs = slice(k*dqk, (k+1)*dqk), slice(k*dv, (k+1)*dv)
            Qk, Kk, Vk = Q[s:e, qs], K[s:e, qs], V[s:e, vs]
            S = Qk@Kk.T + W["rab_pos"][k][pb] + W["rab_time"][k][tb]
            A = np.where(causal, F.silu(S), 0.0)
            dOk = dO[s:e, vs]
            dA = np.where(causal, dOk@Vk.T/n, 0.0)
            Pm = A/n
            if 'P' in R: Pm = f16(Pm)
            dV[s:e, vs] += Pm.T@dOk
            dS = np.where(causal, dA*BW.silu_grad(S), 0.0)
            if 'dS' in R: dS = f16(dS)
            dQ[s:e, qs] += dS@Kk; dK[s:e, qs] += dS.T@Qk
    dG = np.concatenate([dU, dV, dQ, dK], 1)
    dP = dG*BW.silu_grad(Pq)
    if 'dP' in R: dP = f16(dP)
    g["dW1"] = dP.T@X; g["db1"] = dP.sum(0)
    dX += dP@W["W1"]
    g["dX"] = dX
    return g

dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
w = hw.custom("bwdstack", [300, 129, 1, 64, 0, 200], dims, n_layers=2, seed=82)
dY = hw.round_to_bf16(np.random.default_rng(83).standard_normal(w.X.shape).astype(np.float32))
# layer 1 (top) alone, with its real input
X1 = F.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
ref = BW.layer_bwd(X1, w.offsets, w.timestamps, w.weights[1], dims, dY)
allR = ['pre','G','xn','gyh','Z','dO','P','dS','dP','fwdP']
for R in []:
    g = layer_bwd_emu(X1, w.offsets, w.timestamps, w.weights[1], dims, dY, set(R))
    print(R, 'dX %.2e rms %.2e' % (relerr(g['dX'], ref['dX']), rmserr(g['dX'], ref['dX'])),
          'dW1 %.2e' % relerr(g['dW1'], ref['dW1']))

for D in (64, 128):
    dims = hw.LayerDims(128, 2, D, D, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom(f"bwd{D}", [1, 127, 128, 129, 300, 0, 5, 257], dims, seed=80 + D)
    dY = hw.round_to_bf16(np.random.default_rng(81).standard_normal(w.X.shape).astype(np.float32))
    ref = BW.layer_bwd(w.X, w.offsets, w.timestamps, w.weights[0], dims, dY)
    g = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, dY, set(allR))
    print('single D', D, {k: '%.2e' % relerr(g[k], ref[k]) for k in ref if k in g})

def layer_fwd_emu(X, off, ts, w, dims):
    # the GPU forward: fp16 G, fp16 P in attention, normalised O in fp16, fp16 Z, fp16 output stream
    X = np.asarray(X, np.float64)
    W = {k: np.asarray(v, np.float64) for k, v in w.items()}
    h, dqk, dv = dims.n_heads, dims.d_qk, dims.d_v
    G = f16(F.silu(X @ W["W1"].T + W["b1"]))
    parts = F.split_uvqk(G, dims); U, V, Q, K = parts["U"], parts["V"], parts["Q"], parts["K"]
    T = X.shape[0]; O = np.zeros((T, h*dv))
    for b in range(len(off)-1):
        s, e = int(off[b]), int(off[b+1]); n = e - s
        if n == 0: continue
        i = np.arange(n); dist = i[:, None]-i[None, :]; causal = dist >= 0
        pb = F.log_bucket(np.where(causal, dist, 0), dims.n_pos_buckets, dims.pos_sub_bits)
        t = ts[s:e]; tb = F.log_bucket(np.maximum(t[:, None]-t[None, :], 0), dims.n_time_buckets, dims.time_sub_bits)
        for k in range(h):
            qs, vs = slice(k*dqk, (k+1)*dqk), slice(k*dv, (k+1)*dv)
            S = Q[s:e, qs]@K[s:e, qs].T + W["rab_pos"][k][pb] + W["rab_time"][k][tb]
            A = np.where(causal, f16(F.silu(S)), 0.0)
            O[s:e, vs] = A@V[s:e, vs]/n
    Z = f16(F.layer_norm(O, W["ln_gamma"], W["ln_beta"], dims.ln_eps) * U)
    return f16(X + Z @ W["W2"].T + W["b2"])

dims = hw.LayerDims(256, 2, 128, 128, 128, 128, 4, 2, 1e-6, hw.BF16)
w = hw.custom("bwdstack", [300, 129, 1, 64, 0, 200], dims, n_layers=2, seed=82)
dY = hw.round_to_bf16(np.random.default_rng(83).standard_normal(w.X.shape).astype(np.float32))
ref_dX, ref = BW.stack_bwd(w.X, w.offsets, w.timestamps, w.weights, dims, dY)
X1 = layer_fwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims)
g1 = layer_bwd_emu(X1, w.offsets, w.timestamps, w.weights[1], dims, dY, set(allR))
g0 = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, g1['dX'], set(allR))
print('stack emu dX', '%.2e' % relerr(g0['dX'], ref_dX))
for l, g in ((0, g0), (1, g1)):
    print(l, {k: '%.2e' % relerr(g[k], ref[l][k]) for k in ref[l] if k in g})
X1e = F.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
g1 = layer_bwd_emu(X1e, w.offsets, w.timestamps, w.weights[1], dims, dY, set(allR))
g0 = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, g1['dX'], set(allR))
print('exact-X1 stack emu dX', '%.2e' % relerr(g0['dX'], ref_dX), 'dW1[0] %.2e' % relerr(g0['dW1'], ref[0]['dW1']))
g1 = layer_bwd_emu(X1, w.offsets, w.timestamps, w.weights[1], dims, dY, set())
g0 = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, g1['dX'], set())
print('gpu-X1, exact bwd: dX', '%.2e' % relerr(g0['dX'], ref_dX), 'dW1[0] %.2e' % relerr(g0['dW1'], ref[0]['dW1']))
print('X1 err', relerr(X1, X1e))
g1 = layer_bwd_emu(X1e, w.offsets, w.timestamps, w.weights[1], dims, dY, set())
print('gy0 stats: rms %.3e max %.3e' % (np.sqrt((g1['dX']**2).mean()), np.abs(g1['dX']).max()))
for R in [[r] for r in allR]:
    g0 = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, g1['dX'], set(R))
    print(R, 'dX %.2e dW1 %.2e drab? dW2 %.2e' % (relerr(g0['dX'], ref_dX), relerr(g0['dW1'], ref[0]['dW1']), relerr(g0['dW2'], ref[0]['dW2'])))
g1 = layer_bwd_emu(X1e, w.offsets, w.timestamps, w.weights[1], dims, dY, set(allR))
g0 = layer_bwd_emu(w.X, w.offsets, w.timestamps, w.weights[0], dims, g1['dX'], set(allR))
err = np.abs(g0['dX'] - ref_dX).max(1)
print('offsets', w.offsets, 'worst rows', np.argsort(err)[-5:], err[np.argsort(err)[-5:]] / np.sqrt((ref_dX**2).mean()))
# per-layer O spread per row (layer 0)
_, it = F.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims, return_intermediates=True)
sd = it['O'].std(1)
print('sigma(O) at worst rows', sd[np.argsort(err)[-5:]], 'median', np.median(sd))
mask = np.ones(len(err), bool); mask[np.argsort(err)[-1]] = False
print('max err excluding the worst row', err[mask].max() / np.sqrt((ref_dX**2).mean()))
print('rms err', np.sqrt(((g0['dX'] - ref_dX)**2).mean()) / np.sqrt((ref_dX**2).mean()))
