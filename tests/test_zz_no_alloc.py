"""hstu_layer_fwd_noalloc: the layer for callers that cannot allocate device
memory (their allocator belongs to another runtime, or cudaMalloc is off
limits after start-up).  It runs in the library's fixed device scratch
instead of a caller-provided workspace.

Checked through the C ABI on the GPU, three calls in a row on the shared
scratch: a batch, then a smaller batch of another shape and other weights
(state the first call left in the scratch must not leak into the second),
then the first batch again.  Each output equals, bit for bit, the existing
hstu_layer_fwd on the same inputs and weights with a torch-allocated
workspace (the same kernels run), and matches the float64 oracle within the
bf16 bound of the parity tests.  A size whose workspace exceeds the scratch
is rejected before any launch.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest

import hstu_workloads as hw
from gpu_util import TOL, relerr
from oracle import hstu_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def _case(name, lengths, seed):
    import torch
    from hstu_sequential_transducer_layer_b200 import binding as B
    from hstu_sequential_transducer_layer_b200 import HSTURunner

    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom(name, lengths, dims, seed=seed)
    need = B.hstu_workspace_size(B.make_desc(**hw.dims_dict(dims)), 1, w.B, w.T, w.max_len)
    assert need <= B.NOALLOC_SCRATCH_BYTES
    r = HSTURunner(hw.dims_dict(dims), w.weights, "cuda")
    dev = (r.to_device(w.offsets, "i64"), r.to_device(w.X), r.to_device(w.timestamps, "i64"))
    ref = r.stack(dev[0], dev[1], dev[2], w.max_len)   # existing entry point, own workspace
    torch.cuda.synchronize()
    assert r.status() == 0
    oracle = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
    return w, r, dev, ref.view(torch.int16).cpu().numpy(), oracle


def _noalloc(w, r, dev):
    import torch
    from hstu_sequential_transducer_layer_b200 import binding as B

    off, X, ts = dev
    out = torch.full_like(X, float("nan"))
    B.hstu_layer_fwd_noalloc(r.desc, w.B, w.T, w.max_len, off, X, r._warr[0], ts, out)
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_workspace_entry_and_oracle_across_calls():
    big = _case("noalloc_big", [200, 1, 129, 0, 64, 300], seed=90)
    small = _case("noalloc_small", [5, 130, 17], seed=91)
    for w, r, dev, ref_bits, oracle in (big, small, big):
        out = _noalloc(w, r, dev)
        import torch
        assert np.array_equal(out.view(torch.int16).cpu().numpy(), ref_bits), w.name
        assert relerr(out.double().cpu().numpy(), oracle) <= TOL[hw.BF16], w.name


def test_noalloc_rejects_sizes_beyond_scratch():
    from hstu_sequential_transducer_layer_b200 import binding as B

    desc = B.make_desc(1024, 8, 128, 128, 128, 128, 4, 2, 1e-6, "bf16")
    T = 200_000
    assert B.hstu_workspace_size(desc, 1, 1000, T, 1024) > B.NOALLOC_SCRATCH_BYTES
    w = B.LayerWeights(*([0x1000] * 8))
    code = B.lib().hstu_layer_fwd_noalloc(ctypes.byref(desc), 1000, T, 1024, 0x1000, 0x2000,
                                          ctypes.byref(w), 0x3000, 0x4000, None)
    assert code == 3  # HSTU_ERR_WORKSPACE, nothing launched
