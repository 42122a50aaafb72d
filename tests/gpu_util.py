"""Helpers shared by the GPU parity tests: error metrics and running a
workload through the C ABI (via the runner)."""
import math

import numpy as np

import hstu_workloads as hw

# Tolerances: max |gpu - oracle| / RMS(oracle).
TOL = {hw.FP32: 1e-4, hw.BF16: 2e-2}


def relerr(g, r) -> float:
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    rms = math.sqrt(float(np.mean(r * r))) if r.size else 0.0
    if rms == 0.0:
        return float(np.max(np.abs(g - r))) if r.size else 0.0
    return float(np.max(np.abs(g - r))) / rms


def ulp16(r, mant_bits=10):
    """Unit in the last place of |r| for a 16-bit float with `mant_bits`
    stored mantissa bits (fp16: 10, bf16: 7)."""
    a = np.abs(np.asarray(r, np.float64))
    e = np.floor(np.log2(np.maximum(a, 1e-38)))
    return np.exp2(e - mant_bits)


def ulperr(g, r, mant_bits=10, abs_rel=1e-4) -> float:
    """max |g - r| / (ulp(r) + abs_rel * RMS(r)): a stored 16-bit value within
    one ulp of the exact result, plus an absolute floor for values near zero,
    where the fp32 accumulation of the producing GEMM (error ~1e-6 of the
    summed magnitudes) exceeds any ulp of the result."""
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    if not r.size:
        return 0.0
    rms = math.sqrt(float(np.mean(r * r)))
    return float(np.max(np.abs(g - r) / (ulp16(r, mant_bits) + abs_rel * rms)))


def rmserr(g, r) -> float:
    g = np.asarray(g, np.float64)
    r = np.asarray(r, np.float64)
    rms = math.sqrt(float(np.mean(r * r))) or 1.0
    return math.sqrt(float(np.mean((g - r) ** 2))) / rms


def runner_for(w, device="cuda", f16_weights=True):
    from hstu_sequential_transducer_layer_b200 import HSTURunner
    return HSTURunner(hw.dims_dict(w.dims), w.weights, device, f16_weights=f16_weights)


def run_stack(w, n_layers=None, runner=None):
    """Runs the stack on the GPU.  Returns (Y float64 [T,d], runner, device inputs)."""
    import torch
    r = runner or runner_for(w)
    off = r.to_device(w.offsets, "i64")
    X = r.to_device(w.X, "act")
    ts = r.to_device(w.timestamps, "i64")
    out = r.stack(off, X, ts, w.max_len, n_layers=n_layers)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), r, (off, X, ts)


def run_rank(w, microbatch=None, runner=None, candidates=None, cand_offsets=None,
             request_ts="auto"):
    import torch
    r = runner or runner_for(w)
    cands = w.candidates if candidates is None else candidates
    coff = w.cand_offsets if cand_offsets is None else cand_offsets
    req = w.request_ts if isinstance(request_ts, str) else request_ts
    m = np.diff(coff)
    scores = r.rank(r.to_device(w.offsets, "i64"), r.to_device(w.X, "act"),
                    r.to_device(w.timestamps, "i64"), r.to_device(coff, "i64"),
                    r.to_device(cands, "act"),
                    None if req is None else r.to_device(req, "i64"),
                    int(microbatch or w.microbatch), r.to_device(w.head_vec, "act"),
                    w.max_len, int(m.max(initial=0)))
    torch.cuda.synchronize()
    return scores.double().cpu().numpy(), r


def decode_o(o, n_heads: int, d_v: int):
    """The attention output O [T, h*d_v] (float64) from what the layer call
    left in the workspace: fp32 O as is (fp32 path), or, on the tensor-core
    path, (Xn, S) with O = m + s * Xn per (row, head)."""
    if not isinstance(o, tuple):
        return o.double().cpu().numpy()
    xn, st = o
    xn = xn.double().cpu().numpy().reshape(xn.shape[0], n_heads, d_v)
    st = st.double().cpu().numpy()
    return (st[:, :, :1] + st[:, :, 1:] * xn).reshape(xn.shape[0], n_heads * d_v)
