"""ctypes binding of libhstu.so (include/hstu.h), argument marshalling only.

Every function has the name of the C entry point it calls and takes torch
tensors (for device memory) or plain integers.  PyTorch supplies device
memory and the current CUDA stream; every step of the computation runs in
the library's CUDA kernels.  If libhstu.so is missing the first call raises
``HstuError``: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhstu.so")

HSTU_BF16, HSTU_FP32 = 0, 1
STATUS_NAMES = {0: "HSTU_OK", 1: "HSTU_ERR_INVALID_ARG", 2: "HSTU_ERR_UNSUPPORTED",
                3: "HSTU_ERR_WORKSPACE", 4: "HSTU_ERR_CUDA", 5: "HSTU_ERR_BAD_OFFSETS",
                6: "HSTU_ERR_TIMEOUT", 7: "HSTU_ERR_BAD_TIMESTAMPS", 8: "HSTU_ERR_BAD_IDS"}

# Every symbol include/hstu.h declares.
EXPORTED = ["hstu_workspace_size", "hstu_layer_fwd", "hstu_stack_fwd", "hstu_mfalcon_rank",
            "hstu_bwd_workspace_size", "hstu_layer_bwd", "hstu_stack_bwd",
            "hstu_layer_fwd_noalloc", "hstu_sl_embed_workspace_size", "hstu_sl_embed",
            "hstu_sl_keep_count", "hstu_bf16_to_f16", "hstu_retrieval_workspace_size",
            "hstu_retrieval_topk", "hstu_retrieval_fallback_taken",
            "hstu_transformer_workspace_size",
            "hstu_transformer_layer_fwd",
            "hstu_read_status", "hstu_debug_offsets", "hstu_debug_keep_z",
            "hstu_debug_wait_test",
            "hstu_trace_enable", "hstu_trace_only", "hstu_trace_read",
            "hstu_kernel_name", "hstu_launch_count", "hstu_last_error", "hstu_set_option",
            "hstu_status_string",
            "hstu_version"]


class HstuError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.code, self.code)}")


class LayerDesc(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("n_pos_buckets", ctypes.c_int32), ("n_time_buckets", ctypes.c_int32),
                ("pos_sub_bits", ctypes.c_int32), ("time_sub_bits", ctypes.c_int32),
                ("ln_eps", ctypes.c_float), ("dtype", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("ln_gamma", ctypes.c_void_p),
                ("ln_beta", ctypes.c_void_p), ("rab_pos", ctypes.c_void_p),
                ("rab_time", ctypes.c_void_p), ("W1_f16", ctypes.c_void_p),
                ("W2_f16", ctypes.c_void_p)]


GRAD_KEYS = ("dW1", "db1", "dW2", "db2", "dln_gamma", "dln_beta", "drab_pos", "drab_time")


class LayerGrads(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in GRAD_KEYS]


class TransformerWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("ln1_gamma", "ln1_beta", "W_qkv", "W_o", "ln2_gamma",
                                               "ln2_beta", "W_1", "b_1", "W_2", "b_2")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhstu.so (built in-tree by ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise HstuError(4, f"libhstu.so not found at {LIB_PATH}; build it with "
                           "`python -m hstu_sequential_transducer_layer_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    i32, i64, sz, vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
    pdesc = ctypes.POINTER(LayerDesc)
    pw = ctypes.POINTER(LayerWeights)
    L.hstu_workspace_size.argtypes = [pdesc, i32, i64, i64, i64, i64, i64, i32]
    L.hstu_workspace_size.restype = sz
    L.hstu_layer_fwd.argtypes = [pdesc, i64, i64, i64, vp, vp, pw, vp, vp, vp, sz, vp]
    L.hstu_layer_fwd.restype = i32
    L.hstu_stack_fwd.argtypes = [pdesc, i32, pw, i64, i64, i64, vp, vp, vp, vp, vp, sz, vp]
    L.hstu_stack_fwd.restype = i32
    L.hstu_mfalcon_rank.argtypes = [pdesc, i32, pw, i64, i64, i64, vp, vp, vp, i64, i64, vp, vp,
                                    vp, i32, vp, vp, vp, sz, vp]
    L.hstu_mfalcon_rank.restype = i32
    pg = ctypes.POINTER(LayerGrads)
    L.hstu_bwd_workspace_size.argtypes = [pdesc, i32, i64, i64, i64]
    L.hstu_bwd_workspace_size.restype = sz
    L.hstu_layer_bwd.argtypes = [pdesc, pw, i64, i64, i64, vp, vp, vp, vp, vp, pg, vp, sz, vp]
    L.hstu_layer_bwd.restype = i32
    L.hstu_stack_bwd.argtypes = [pdesc, i32, pw, i64, i64, i64, vp, vp, vp, vp, vp, pg, vp, sz, vp]
    L.hstu_stack_bwd.restype = i32
    L.hstu_layer_fwd_noalloc.argtypes = [pdesc, i64, i64, i64, vp, vp, pw, vp, vp, vp]
    L.hstu_layer_fwd_noalloc.restype = i32
    L.hstu_sl_embed_workspace_size.argtypes = []
    L.hstu_sl_embed_workspace_size.restype = sz
    L.hstu_sl_keep_count.argtypes = [i64]
    L.hstu_sl_keep_count.restype = i64
    L.hstu_bf16_to_f16.argtypes = [vp, vp, i64, vp]
    L.hstu_bf16_to_f16.restype = i32
    L.hstu_retrieval_workspace_size.argtypes = [i64, i64, i32, i32, i32]
    L.hstu_retrieval_workspace_size.restype = sz
    L.hstu_retrieval_topk.argtypes = [i64, i64, i32, vp, vp, i64, vp, i32, vp, vp, vp, sz, vp]
    L.hstu_retrieval_topk.restype = i32
    L.hstu_retrieval_fallback_taken.argtypes = [vp, sz, ctypes.POINTER(ctypes.c_int32), vp]
    L.hstu_retrieval_fallback_taken.restype = i32
    L.hstu_transformer_workspace_size.argtypes = [i32, i32, i32, i64, i64]
    L.hstu_transformer_workspace_size.restype = sz
    L.hstu_transformer_layer_fwd.argtypes = [i32, i32, i32, ctypes.c_float,
                                             ctypes.POINTER(TransformerWeights), i64, i64, i64, vp,
                                             vp, vp, vp, sz, vp]
    L.hstu_transformer_layer_fwd.restype = i32
    L.hstu_sl_embed.argtypes = [i64, i64, i64, vp, vp, vp, ctypes.c_uint64, vp, i64, vp, i64, i32,
                                vp, vp, vp, vp, sz, vp]
    L.hstu_sl_embed.restype = i32
    L.hstu_read_status.argtypes = [vp, sz, vp]
    L.hstu_read_status.restype = i32
    L.hstu_debug_offsets.argtypes = [pdesc, i64, i64, i64, ctypes.POINTER(sz),
                                     ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.hstu_debug_offsets.restype = i32
    L.hstu_debug_keep_z.argtypes = [i32]
    L.hstu_debug_keep_z.restype = i32
    L.hstu_debug_wait_test.argtypes = [ctypes.c_uint32, i32]
    L.hstu_debug_wait_test.restype = i32
    L.hstu_trace_enable.argtypes = [i32]
    L.hstu_trace_enable.restype = i32
    L.hstu_trace_only.argtypes = [i32]
    L.hstu_trace_only.restype = i32
    L.hstu_trace_read.argtypes = [ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_float), i32]
    L.hstu_trace_read.restype = i32
    L.hstu_kernel_name.argtypes = [i32]
    L.hstu_kernel_name.restype = ctypes.c_char_p
    L.hstu_launch_count.argtypes = []
    L.hstu_launch_count.restype = i64
    L.hstu_set_option.argtypes = [ctypes.c_char_p, i64]
    L.hstu_set_option.restype = i32
    L.hstu_last_error.argtypes = []
    L.hstu_last_error.restype = ctypes.c_char_p
    L.hstu_status_string.argtypes = [i32]
    L.hstu_status_string.restype = ctypes.c_char_p
    L.hstu_version.argtypes = []
    L.hstu_version.restype = i32
    _lib = L
    return L


# ---------------------------------------------------------------- marshalling
def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _nbytes(t) -> int:
    return int(t.numel() * t.element_size())


def _check(code: int, where: str) -> None:
    if code != 0:
        if code == 4:  # HSTU_ERR_CUDA: name the failing runtime call
            where = f"{where} ({lib().hstu_last_error().decode()})"
        raise HstuError(code, where)


def make_desc(d_model, n_heads, d_qk, d_v, n_pos_buckets, n_time_buckets, pos_sub_bits,
              time_sub_bits, ln_eps=1e-6, dtype="bf16") -> LayerDesc:
    dt = HSTU_BF16 if dtype in ("bf16", HSTU_BF16) else HSTU_FP32
    return LayerDesc(d_model, n_heads, d_qk, d_v, n_pos_buckets, n_time_buckets, pos_sub_bits,
                     time_sub_bits, float(ln_eps), dt)


def weights_struct(w: Dict[str, object]) -> LayerWeights:
    """LayerWeights from a dict of device tensors (W1, b1, W2, b2, ln_gamma,
    ln_beta, rab_pos, rab_time)."""
    return LayerWeights(*[_ptr(w[k]) for k in ("W1", "b1", "W2", "b2", "ln_gamma", "ln_beta",
                                                "rab_pos", "rab_time")],
                        *[_ptr(w[k]) if w.get(k) is not None else None
                          for k in ("W1_f16", "W2_f16")])


def weights_array(ws: Sequence[Dict[str, object]]):
    arr = (LayerWeights * len(ws))()
    for i, w in enumerate(ws):
        arr[i] = weights_struct(w)
    return arr


def weights_to_device(weights: Sequence[Dict[str, np.ndarray]], dtype: str, device) -> List[Dict]:
    """Copy a list of per-layer numpy weight dicts to the device (dense
    weights in the layer dtype, rab tables fp32)."""
    import torch
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = []
    for w in weights:
        d = {}
        for k in ("W1", "b1", "W2", "b2", "ln_gamma", "ln_beta"):
            d[k] = torch.from_numpy(np.ascontiguousarray(w[k], np.float32)).to(device=device, dtype=tdt)
        for k in ("rab_pos", "rab_time"):
            d[k] = torch.from_numpy(np.ascontiguousarray(w[k], np.float32)).to(device)
        out.append(d)
    return out


# ---------------------------------------------------------------- entry points
def hstu_workspace_size(desc: LayerDesc, n_layers: int, B: int, total_tokens: int, max_len: int,
                        total_cands: int = 0, max_cands: int = 0, microbatch: int = 0) -> int:
    n = lib().hstu_workspace_size(ctypes.byref(desc), n_layers, B, total_tokens, max_len,
                                  total_cands, max_cands, microbatch)
    if n == 0:
        raise HstuError(1, "hstu_workspace_size")
    return int(n)


def hstu_layer_fwd(desc, B, total_tokens, max_len, offsets, X, weights, timestamps, out,
                   workspace, stream=None) -> None:
    ws = weights if isinstance(weights, LayerWeights) else weights_struct(weights)
    _check(lib().hstu_layer_fwd(ctypes.byref(desc), B, total_tokens, max_len, _ptr(offsets),
                                _ptr(X), ctypes.byref(ws), _ptr(timestamps), _ptr(out),
                                _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "hstu_layer_fwd")


NOALLOC_SCRATCH_BYTES = 64 << 20  # HSTU_NOALLOC_SCRATCH_BYTES


def hstu_layer_fwd_noalloc(desc, B, total_tokens, max_len, offsets, X, weights, timestamps, out,
                           stream=None) -> None:
    """One layer in the library's fixed device scratch (no workspace argument)."""
    ws = weights if isinstance(weights, LayerWeights) else weights_struct(weights)
    _check(lib().hstu_layer_fwd_noalloc(ctypes.byref(desc), B, total_tokens, max_len,
                                        _ptr(offsets), _ptr(X), ctypes.byref(ws),
                                        _ptr(timestamps), _ptr(out), _stream(stream)),
           "hstu_layer_fwd_noalloc")


def hstu_sl_embed_workspace_size() -> int:
    return int(lib().hstu_sl_embed_workspace_size())


def hstu_bf16_to_f16(src, dst, stream=None) -> None:
    """fp16 copy of a bf16 device tensor (same shape) through the library."""
    _check(lib().hstu_bf16_to_f16(_ptr(src), _ptr(dst), int(src.numel()), _stream(stream)),
           "hstu_bf16_to_f16")


def hstu_retrieval_workspace_size(n_users, n_items, d, K, from_rows=False) -> int:
    n = lib().hstu_retrieval_workspace_size(n_users, n_items, d, K, 1 if from_rows else 0)
    if n == 0:
        raise HstuError(1, "hstu_retrieval_workspace_size")
    return int(n)


def hstu_retrieval_topk(H, E, K, out_scores, out_ids, workspace, user_offsets=None,
                        n_users=None, stream=None) -> None:
    """Top-K catalog items per user (see include/hstu.h).  H: bf16 [n_users, d]
    user vectors, or with user_offsets the encoder output [rows, d]; E: bf16
    [n_items, d]."""
    U = int(n_users if n_users is not None else
            (user_offsets.numel() - 1 if user_offsets is not None else H.shape[0]))
    rows = int(H.shape[0]) if user_offsets is not None else 0
    _check(lib().hstu_retrieval_topk(U, int(E.shape[0]), int(E.shape[1]), _ptr(H),
                                     _ptr(user_offsets), rows, _ptr(E), int(K), _ptr(out_scores),
                                     _ptr(out_ids), _ptr(workspace), _nbytes(workspace),
                                     _stream(stream)),
           "hstu_retrieval_topk")


def hstu_retrieval_fallback_taken(workspace, stream=None) -> bool:
    v = ctypes.c_int32(0)
    _check(lib().hstu_retrieval_fallback_taken(_ptr(workspace), _nbytes(workspace),
                                               ctypes.byref(v), _stream(stream)),
           "hstu_retrieval_fallback_taken")
    return bool(v.value)


def hstu_transformer_workspace_size(d_model, n_heads, d_ff, B, total_tokens) -> int:
    n = lib().hstu_transformer_workspace_size(d_model, n_heads, d_ff, B, total_tokens)
    if n == 0:
        raise HstuError(1, "hstu_transformer_workspace_size")
    return int(n)


def hstu_transformer_layer_fwd(d_model, n_heads, d_ff, ln_eps, weights, B, total_tokens, max_len,
                               offsets, X, out, workspace, stream=None) -> None:
    """The softmax-Transformer comparator layer (see include/hstu.h); `weights`
    is a TransformerWeights struct or a dict of device tensors."""
    if not isinstance(weights, TransformerWeights):
        weights = TransformerWeights(*[_ptr(weights[k]) for k, _ in TransformerWeights._fields_])
    _check(lib().hstu_transformer_layer_fwd(d_model, n_heads, d_ff, float(ln_eps),
                                            ctypes.byref(weights), B, total_tokens, max_len,
                                            _ptr(offsets), _ptr(X), _ptr(out), _ptr(workspace),
                                            _nbytes(workspace), _stream(stream)),
           "hstu_transformer_layer_fwd")


def hstu_sl_keep_count(n: int) -> int:
    return int(lib().hstu_sl_keep_count(int(n)))


def hstu_sl_embed(B, raw_total, max_raw_len, raw_offsets, raw_ids, raw_timestamps, seed,
                  content_table, action_table, out_offsets, out_X, out_timestamps, workspace,
                  stream=None) -> None:
    """Stochastic Length + token embedding on the device (see include/hstu.h);
    the tables are bf16 [rows, d] device tensors."""
    _check(lib().hstu_sl_embed(B, raw_total, max_raw_len, _ptr(raw_offsets), _ptr(raw_ids),
                               _ptr(raw_timestamps), int(seed) & ((1 << 64) - 1),
                               _ptr(content_table), int(content_table.shape[0]),
                               _ptr(action_table), int(action_table.shape[0]),
                               int(content_table.shape[1]), _ptr(out_offsets), _ptr(out_X),
                               _ptr(out_timestamps), _ptr(workspace), _nbytes(workspace),
                               _stream(stream)),
           "hstu_sl_embed")


def hstu_stack_fwd(desc, n_layers, weights, B, total_tokens, max_len, offsets, X, timestamps,
                   out, workspace, stream=None) -> None:
    arr = weights if not isinstance(weights, (list, tuple)) else weights_array(weights)
    _check(lib().hstu_stack_fwd(ctypes.byref(desc), n_layers, arr, B, total_tokens, max_len,
                                _ptr(offsets), _ptr(X), _ptr(timestamps), _ptr(out),
                                _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "hstu_stack_fwd")


def grads_array(gs: Sequence[Dict[str, object]]):
    """LayerGrads array from per-layer dicts of fp32 device tensors."""
    arr = (LayerGrads * len(gs))()
    for i, g in enumerate(gs):
        arr[i] = LayerGrads(*[_ptr(g[k]) for k in GRAD_KEYS])
    return arr


def hstu_bwd_workspace_size(desc: LayerDesc, n_layers: int, B: int, total_tokens: int,
                            max_len: int) -> int:
    n = int(lib().hstu_bwd_workspace_size(ctypes.byref(desc), n_layers, B, total_tokens, max_len))
    if n == 0:
        raise HstuError(1, "hstu_bwd_workspace_size")
    return n


def hstu_layer_bwd(desc, weights, B, total_tokens, max_len, offsets, X, timestamps, dY, dX,
                   grads, workspace, stream=None) -> None:
    w = weights if isinstance(weights, LayerWeights) else weights_struct(weights)
    g = grads if not isinstance(grads, (list, tuple)) else grads_array(grads)
    _check(lib().hstu_layer_bwd(ctypes.byref(desc), ctypes.byref(w), B, total_tokens, max_len,
                                _ptr(offsets), _ptr(X), _ptr(timestamps), _ptr(dY), _ptr(dX), g,
                                _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "hstu_layer_bwd")


def hstu_stack_bwd(desc, n_layers, weights, B, total_tokens, max_len, offsets, X, timestamps, dY,
                   dX, grads, workspace, stream=None) -> None:
    arr = weights if not isinstance(weights, (list, tuple)) else weights_array(weights)
    g = grads if not isinstance(grads, (list, tuple)) else grads_array(grads)
    _check(lib().hstu_stack_bwd(ctypes.byref(desc), n_layers, arr, B, total_tokens, max_len,
                                _ptr(offsets), _ptr(X), _ptr(timestamps), _ptr(dY), _ptr(dX), g,
                                _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "hstu_stack_bwd")


def hstu_mfalcon_rank(desc, n_layers, weights, B, total_hist, max_len, hist_offsets, history,
                      hist_timestamps, total_cands, max_cands, cand_offsets, candidates,
                      request_ts, microbatch, head_vec, scores, workspace, stream=None) -> None:
    arr = weights if not isinstance(weights, (list, tuple)) else weights_array(weights)
    _check(lib().hstu_mfalcon_rank(ctypes.byref(desc), n_layers, arr, B, total_hist, max_len,
                                   _ptr(hist_offsets), _ptr(history), _ptr(hist_timestamps),
                                   total_cands, max_cands, _ptr(cand_offsets), _ptr(candidates),
                                   _ptr(request_ts), microbatch, _ptr(head_vec), _ptr(scores),
                                   _ptr(workspace), _nbytes(workspace), _stream(stream)),
           "hstu_mfalcon_rank")


def hstu_read_status(workspace, stream=None) -> int:
    return int(lib().hstu_read_status(_ptr(workspace), _nbytes(workspace), _stream(stream)))


def hstu_debug_offsets(desc, B, total_tokens, max_len):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().hstu_debug_offsets(ctypes.byref(desc), B, total_tokens, max_len,
                                    ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "hstu_debug_offsets")
    return int(a.value), int(b.value), int(c.value)


def hstu_set_option(name: str, value: int) -> None:
    _check(lib().hstu_set_option(name.encode(), int(value)), "hstu_set_option")


def hstu_debug_keep_z(on: bool) -> None:
    _check(lib().hstu_debug_keep_z(1 if on else 0), "hstu_debug_keep_z")


def hstu_debug_wait_test(wait_limit_us: int, inject_stall: int) -> None:
    _check(lib().hstu_debug_wait_test(int(wait_limit_us), int(inject_stall)),
           "hstu_debug_wait_test")


def hstu_trace_enable(max_records: int) -> None:
    _check(lib().hstu_trace_enable(max_records), "hstu_trace_enable")


def hstu_trace_only(kernel_id: int) -> None:
    _check(lib().hstu_trace_only(kernel_id), "hstu_trace_only")


def hstu_trace_read(capacity: int = 1 << 16):
    ids = (ctypes.c_int32 * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = lib().hstu_trace_read(ids, ms, capacity)
    return [(int(ids[i]), float(ms[i])) for i in range(n)]


def hstu_kernel_name(kernel_id: int) -> str:
    return lib().hstu_kernel_name(kernel_id).decode()


def hstu_launch_count() -> int:
    return int(lib().hstu_launch_count())


def hstu_status_string(code: int) -> str:
    return lib().hstu_status_string(code).decode()


def hstu_version() -> int:
    return int(lib().hstu_version())
