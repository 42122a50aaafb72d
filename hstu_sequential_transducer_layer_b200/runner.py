"""Holds a layer descriptor, device weights and a reusable workspace, and
calls the C ABI with them.  Allocation (weights, workspace, outputs) goes
through torch; the computation is the library's."""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

from . import binding as _b


class HSTURunner:
    def __init__(self, dims: Dict[str, object], weights: Sequence[Dict[str, np.ndarray]],
                 device="cuda", f16_weights: bool = True):
        """`f16_weights` (bf16 layers): make the fp16 copies of W1 (layers
        >= 1) and W2 that the tensor-core path multiplies once, here, instead
        of in every call."""
        import torch
        self.torch = torch
        self.device = torch.device(device)
        self.dtype = str(dims["dtype"])
        self.tdtype = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        self.desc = _b.make_desc(int(dims["d_model"]), int(dims["n_heads"]), int(dims["d_qk"]),
                                 int(dims["d_v"]), int(dims["n_pos_buckets"]),
                                 int(dims["n_time_buckets"]), int(dims["pos_sub_bits"]),
                                 int(dims["time_sub_bits"]), float(dims["ln_eps"]), self.dtype)
        self.weights = _b.weights_to_device(weights, self.dtype, self.device)
        self.n_layers = len(self.weights)
        if f16_weights and self.dtype == "bf16":
            for l, w in enumerate(self.weights):
                for k in (("W1", "W2") if l > 0 else ("W2",)):
                    w[k + "_f16"] = torch.empty(w[k].shape, dtype=torch.float16,
                                                device=self.device)
                    _b.hstu_bf16_to_f16(w[k], w[k + "_f16"])
        self._warr = _b.weights_array(self.weights)
        self._ws = None

    # ------------------------------------------------------------ memory
    def workspace(self, nbytes: int):
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = self.torch.empty(max(nbytes, 256), dtype=self.torch.uint8, device=self.device)
        return self._ws

    def to_device(self, a: np.ndarray, kind: str = "act"):
        t = self.torch
        if kind == "act":
            return t.from_numpy(np.ascontiguousarray(a, np.float32)).to(self.device, self.tdtype)
        if kind == "i64":
            return t.from_numpy(np.ascontiguousarray(a, np.int64)).to(self.device)
        return t.from_numpy(np.ascontiguousarray(a, np.float32)).to(self.device)

    # ------------------------------------------------------------ calls
    def stack(self, offsets, X, timestamps, max_len: int, n_layers: Optional[int] = None,
              out=None, stream=None):
        """hstu_stack_fwd over device tensors; returns `out`."""
        L = self.n_layers if n_layers is None else n_layers
        B = offsets.numel() - 1
        T = X.shape[0]
        if out is None:
            out = self.torch.empty_like(X)
        nb = _b.hstu_workspace_size(self.desc, L, B, T, max_len)
        ws = self.workspace(nb)
        if L == 1:
            _b.hstu_layer_fwd(self.desc, B, T, max_len, offsets, X, self._warr[0], timestamps, out,
                              ws, stream)
        else:
            _b.hstu_stack_fwd(self.desc, L, self._warr, B, T, max_len, offsets, X, timestamps, out,
                              ws, stream)
        return out

    def kept_sizes(self, raw_lengths) -> tuple:
        """(total, max) of the Stochastic Length keep counts of raw streams of
        the given lengths, from the library's host keep count."""
        k = [_b.hstu_sl_keep_count(int(n)) for n in raw_lengths]
        if any(x < 0 for x in k):
            raise _b.HstuError(2, "hstu_sl_keep_count")
        return int(sum(k)), int(max(k, default=0))

    def stack_raw(self, raw_lengths, raw_offsets, raw_ids, raw_ts, seed: int, content_table,
                  action_table, max_raw_len: int, out=None, stream=None, kept=None):
        """Raw token streams -> Stochastic Length + token embedding
        (hstu_sl_embed) -> the layer stack (hstu_stack_fwd), all on `stream`
        with no host synchronisation.  `raw_lengths` (host) sizes the kept
        batch (or `kept` = kept_sizes(raw_lengths), computed once by the
        caller); the device tensors carry the data.  Returns (out, kept
        offsets, kept timestamps)."""
        t = self.torch
        B = raw_offsets.numel() - 1
        R = raw_ids.numel()
        T, max_len = kept if kept is not None else self.kept_sizes(raw_lengths)
        d = int(content_table.shape[1])
        key = (B, T, d)
        if getattr(self, "_sl_key", None) != key:
            self._sl_key = key
            self._sl_off = t.empty(B + 1, dtype=t.int64, device=self.device)
            self._sl_X = t.empty(max(T, 1), d, dtype=t.bfloat16, device=self.device)
            self._sl_ts = t.empty(max(T, 1), dtype=t.int64, device=self.device)
            self._sl_ws = t.empty(_b.hstu_sl_embed_workspace_size(), dtype=t.uint8,
                                  device=self.device)
        _b.hstu_sl_embed(B, R, max_raw_len, raw_offsets, raw_ids, raw_ts, seed, content_table,
                         action_table, self._sl_off, self._sl_X, self._sl_ts, self._sl_ws, stream)
        X = self._sl_X[:T]
        if out is None:
            out = t.empty_like(X)
        self.stack(self._sl_off, X, self._sl_ts[:T], max_len, out=out, stream=stream)
        return out, self._sl_off, self._sl_ts[:T]

    def sl_status(self, stream=None) -> int:
        return _b.hstu_read_status(self._sl_ws, stream)

    def rank(self, hist_offsets, history, hist_ts, cand_offsets, candidates, request_ts,
             microbatch: int, head_vec, max_len: int, max_cands: int, scores=None, stream=None):
        B = hist_offsets.numel() - 1
        T = history.shape[0]
        C = candidates.shape[0]
        if scores is None:
            scores = self.torch.empty(C, dtype=self.torch.float32, device=self.device)
        nb = _b.hstu_workspace_size(self.desc, self.n_layers, B, T, max_len, C, max_cands,
                                    microbatch)
        ws = self.workspace(nb)
        _b.hstu_mfalcon_rank(self.desc, self.n_layers, self._warr, B, T, max_len, hist_offsets,
                             history, hist_ts, C, max_cands, cand_offsets, candidates, request_ts,
                             microbatch, head_vec, scores, ws, stream)
        return scores

    def status(self, stream=None) -> int:
        return _b.hstu_read_status(self._ws, stream)

    def stack_bwd(self, offsets, X, timestamps, dY, max_len: int, n_layers: Optional[int] = None,
                  dX=None, grads=None, stream=None):
        """hstu_stack_bwd (hstu_layer_bwd for one layer): the gradient dX of a
        loss with respect to X given its gradient dY with respect to the
        stack's output, and every layer's parameter gradients (fp32).
        Returns (dX, [dict per layer])."""
        t = self.torch
        L = self.n_layers if n_layers is None else n_layers
        B = offsets.numel() - 1
        T = X.shape[0]
        d = self.desc
        F = 2 * d.n_heads * (d.d_v + d.d_qk)
        hdv = d.n_heads * d.d_v
        if dX is None:
            dX = t.empty_like(X)
        if grads is None:
            shapes = dict(dW1=(F, d.d_model), db1=(F,), dW2=(d.d_model, hdv), db2=(d.d_model,),
                          dln_gamma=(hdv,), dln_beta=(hdv,),
                          drab_pos=(d.n_heads, d.n_pos_buckets),
                          drab_time=(d.n_heads, d.n_time_buckets))
            grads = [{k: t.empty(v, dtype=t.float32, device=self.device) for k, v in shapes.items()}
                     for _ in range(L)]
        nb = _b.hstu_bwd_workspace_size(self.desc, L, B, T, max_len)
        if getattr(self, "_bws", None) is None or self._bws.numel() < nb:
            self._bws = t.empty(max(nb, 256), dtype=t.uint8, device=self.device)
        if L == 1:
            _b.hstu_layer_bwd(self.desc, self._warr[0], B, T, max_len, offsets, X, timestamps, dY,
                              dX, grads, self._bws, stream)
        else:
            _b.hstu_stack_bwd(self.desc, L, self._warr, B, T, max_len, offsets, X, timestamps, dY,
                              dX, grads, self._bws, stream)
        return dX, grads

    def bwd_status(self, stream=None) -> int:
        return _b.hstu_read_status(self._bws, stream)

    def intermediates(self, B: int, T: int, max_len: int):
        """Views of the f1 output, the attention output and Z that the last
        layer call left in the workspace (see hstu_debug_offsets).  fp32 path:
        (f1, O, Z), all fp32.  Tensor-core (bf16) path: (f1 fp16, (Xn, S), Z
        fp16) where Xn [T, h*d_v] fp16 holds (O - m) / s per (row, head) and S
        [T, h, 2] fp32 the (m, s) pairs; Z is there only while
        hstu_debug_keep_z(1) was in effect."""
        f1o, oo, zo = _b.hstu_debug_offsets(self.desc, B, T, max_len)
        d = self.desc
        F = 2 * d.n_heads * (d.d_v + d.d_qk)
        hdv = d.n_heads * d.d_v
        t = self.torch
        ws = self._ws

        def view(off, cols, dt, size):
            return ws[off:off + T * cols * size].view(dt).view(T, cols)
        if self.dtype != "bf16":
            return view(f1o, F, t.float32, 4), view(oo, hdv, t.float32, 4), view(zo, hdv, t.float32, 4)
        so = oo + ((T * hdv * 2 + 255) // 256) * 256
        stats = view(so, 2 * d.n_heads, t.float32, 4).view(T, d.n_heads, 2)
        return (view(f1o, F, t.float16, 2), (view(oo, hdv, t.float16, 2), stats),
                view(zo, hdv, t.float16, 2))


class TransformerRunner:
    """Device weights and a workspace for the softmax-Transformer comparator
    layer (hstu_transformer_layer_fwd).  Dense weights go to the device as
    fp16, LayerNorm parameters and biases as bf16."""

    DENSE = ("W_qkv", "W_o", "W_1", "W_2")

    def __init__(self, d_model: int, n_heads: int, d_ff: int, weights: Dict[str, np.ndarray],
                 ln_eps: float = 1e-6, device="cuda"):
        import torch
        self.torch = torch
        self.device = torch.device(device)
        self.d, self.h, self.ff, self.eps = int(d_model), int(n_heads), int(d_ff), float(ln_eps)
        self.w = {}
        for k, v in weights.items():
            dt = torch.float16 if k in self.DENSE else torch.bfloat16
            self.w[k] = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(self.device, dt)
        self._struct = _b.TransformerWeights(*[_b._ptr(self.w[k]) for k, _ in
                                               _b.TransformerWeights._fields_])
        self._ws = None

    def layer(self, offsets, X, max_len: int, out=None, stream=None):
        t = self.torch
        B = offsets.numel() - 1
        T = X.shape[0]
        if out is None:
            out = t.empty_like(X)
        nb = _b.hstu_transformer_workspace_size(self.d, self.h, self.ff, B, T)
        if self._ws is None or self._ws.numel() < nb:
            self._ws = t.empty(nb, dtype=t.uint8, device=self.device)
        _b.hstu_transformer_layer_fwd(self.d, self.h, self.ff, self.eps, self._struct, B, T,
                                      max_len, offsets, X, out, self._ws, stream)
        return out

    def status(self, stream=None) -> int:
        return _b.hstu_read_status(self._ws, stream)
