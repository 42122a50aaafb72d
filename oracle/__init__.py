"""CPU float64 oracle for the HSTU layer stack and M-FALCON ranking.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the CUDA path.
"""
from . import hstu_oracle  # noqa: F401
from .hstu_oracle import (  # noqa: F401
    layer_fwd, stack_fwd, layer_rows, stack_user, mfalcon_rank, mfalcon_user,
    log_bucket, silu, layer_norm, split_uvqk,
)
