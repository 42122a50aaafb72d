"""Failure detection of the bounded in-kernel waits, on the GPU, without a
fault: a wait that a test makes run out.

Every wait inside the attention kernel gives up after a bound (1 s by
default), raises HSTU_ERR_TIMEOUT in the call's status word and lets the
kernel wind down: loads in flight land, tensor memory is released, the CTA
returns.  The test hook ``hstu_debug_wait_test`` shortens the bound to 1 ms
for the next attention launch and makes that launch's first CTA stop handing
out work after two items without telling its other roles; they then wait for
a third item that never comes.  No load is skipped, no address is bad, and
nothing traps: the waits simply run out.

Checked: the stalled call returns with status 6 (HSTU_ERR_TIMEOUT); the next
normal call on the same workspace returns status 0 (its kernels could start,
allocate tensor memory and finish, so the stalled launch released it) and
gives the same bits as a call made before the stall, which matches the
oracle within the bf16 bound."""
import numpy as np
import pytest

import hstu_workloads as hw
from gpu_util import TOL, relerr, run_stack
from oracle import hstu_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hstu_sequential_transducer_layer_b200.build import build
    build()


def test_wait_that_runs_out_sets_timeout_and_next_call_is_clean():
    import torch
    from hstu_sequential_transducer_layer_b200 import binding as B

    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    # 96 users x 640 rows: 5 query tiles x 2 heads each = 960 work items, so
    # the first CTA certainly holds two items when the stall is injected
    w = hw.custom("stall", [640] * 96, dims, seed=61)
    Y0, r, (off, X, ts) = run_stack(w)
    assert r.status() == 0

    B.hstu_debug_wait_test(1000, 1)        # 1 ms bound, stall CTA 0 after two items
    r.stack(off, X, ts, w.max_len)
    torch.cuda.synchronize()
    assert r.status() == 6                 # HSTU_ERR_TIMEOUT

    Y1 = r.stack(off, X, ts, w.max_len)    # defaults again, same workspace
    torch.cuda.synchronize()
    assert r.status() == 0
    assert np.array_equal(Y1.double().cpu().numpy(), Y0)

    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
    assert relerr(Y0, ref) <= TOL[hw.BF16]


def test_wait_hook_is_one_shot_and_checks_its_argument():
    from hstu_sequential_transducer_layer_b200 import binding as B

    with pytest.raises(B.HstuError):
        B.hstu_debug_wait_test(1000, 2)
    dims = hw.LayerDims(128, 2, 64, 64, 64, 128, 3, 2, 1e-6, hw.BF16)
    w = hw.custom("stall_once", [300, 129, 1], dims, seed=62)
    # a short bound alone, with no stall: the launch finishes well inside it
    B.hstu_debug_wait_test(200_000, 0)
    Y, r, _ = run_stack(w)
    assert r.status() == 0
    ref = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
    assert relerr(Y, ref) <= TOL[hw.BF16]
