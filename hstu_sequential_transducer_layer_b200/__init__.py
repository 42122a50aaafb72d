"""HSTU layer stack + M-FALCON ranking on one B200 (sm_100a).

The computation lives in ``libhstu.so`` (CUDA kernels behind the C ABI of
``include/hstu.h``); ``binding`` marshals torch tensors into those calls and
``runner`` holds device weights and workspaces for repeated calls.
"""
from .binding import (  # noqa: F401
    HstuError, LayerDesc, LayerWeights, make_desc, weights_struct, weights_array,
    weights_to_device, hstu_workspace_size, hstu_layer_fwd, hstu_stack_fwd, hstu_mfalcon_rank,
    hstu_sl_embed, hstu_sl_embed_workspace_size, hstu_sl_keep_count,
    hstu_bf16_to_f16, hstu_retrieval_workspace_size, hstu_retrieval_topk, hstu_retrieval_fallback_taken,
    hstu_transformer_workspace_size, hstu_transformer_layer_fwd, TransformerWeights,
    hstu_read_status, hstu_debug_offsets, hstu_trace_enable, hstu_trace_only, hstu_trace_read,
    hstu_kernel_name,
    hstu_launch_count, hstu_status_string, hstu_version, lib, LIB_PATH, EXPORTED,
    LayerGrads, grads_array, hstu_bwd_workspace_size, hstu_layer_bwd, hstu_stack_bwd,
    hstu_set_option, hstu_debug_keep_z, hstu_debug_wait_test,
)
from .runner import HSTURunner, TransformerRunner  # noqa: F401,E402
