"""hstu_layer_fwd_noalloc: the layer for callers that cannot allocate device
memory (their allocator belongs to another runtime, or cudaMalloc is off
limits after start-up).  It runs in the library's fixed device scratch
instead of a caller-provided workspace.

Checked through the C ABI on the GPU: two calls in a row match the existing
hstu_layer_fwd (which gets a torch-allocated workspace) within the bf16
tolerance of the parity tests, and a size whose workspace exceeds the scratch
is rejected before any launch.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest

import hstu_workloads as hw
from gpu_util import TOL, relerr

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def test_noalloc_matches_workspace_entry_twice():
    import torch
    from hstu_sequential_transducer_layer_b200 import binding as B
    from hstu_sequential_transducer_layer_b200 import HSTURunner

    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("noalloc", [200, 1, 129, 0, 64], dims, seed=90)
    need = B.hstu_workspace_size(B.make_desc(**{k: v for k, v in hw.dims_dict(dims).items()}),
                                 1, w.B, w.T, w.max_len)
    assert need <= B.NOALLOC_SCRATCH_BYTES

    r = HSTURunner(hw.dims_dict(dims), w.weights, "cuda")
    off, ts, X = r.to_device(w.offsets, "i64"), r.to_device(w.timestamps, "i64"), r.to_device(w.X)
    ref = r.stack(off, X, ts, w.max_len)            # existing entry point, own workspace
    torch.cuda.synchronize()
    assert r.status() == 0
    ref = ref.double().cpu().numpy()

    for _ in range(2):                               # two calls in a row share the scratch
        out = torch.full_like(X, float("nan"))
        B.hstu_layer_fwd_noalloc(r.desc, w.B, w.T, w.max_len, off, X, r._warr[0], ts, out)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert relerr(got, ref) <= TOL[hw.BF16]


def test_noalloc_rejects_sizes_beyond_scratch():
    from hstu_sequential_transducer_layer_b200 import binding as B

    desc = B.make_desc(1024, 8, 128, 128, 128, 128, 4, 2, 1e-6, "bf16")
    T = 200_000
    assert B.hstu_workspace_size(desc, 1, 1000, T, 1024) > B.NOALLOC_SCRATCH_BYTES
    w = B.LayerWeights(*([0x1000] * 8))
    code = B.lib().hstu_layer_fwd_noalloc(ctypes.byref(desc), 1000, T, 1024, 0x1000, 0x2000,
                                          ctypes.byref(w), 0x3000, 0x4000, None)
    assert code == 3  # HSTU_ERR_WORKSPACE, nothing launched
