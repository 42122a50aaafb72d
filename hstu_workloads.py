"""Seeded synthetic inputs for the HSTU layer / M-FALCON workloads.

This module only draws random inputs and rounds them to the storage precision.
It holds none of the layer's arithmetic: both the float64 oracle (``oracle/``)
and the CUDA path (``hstu_sequential_transducer_layer_b200``) receive the same
arrays from here, and neither side imports the other.

Workloads (sizes follow the pages' own workloads, see the docstring of each):

* ``tiny_fp32``      1 layer, B=4, lengths U{8..64}, d=64, 2 heads, 32/32, fp32.
* ``single_layer``   1 layer, B=64, lognormal lengths (median 256, cap 1024),
                     d=256, 4 heads, 64/64, bf16.
* ``long_history``   1 layer, B=16, lengths U{2048..8192}, d=512, 8 heads,
                     64/64, bf16 (~80k tokens; the 8,192-token, d=512, 8-head
                     encoder of 'HSTUとGenerative Recommenders', section
                     'Production評価の12.4%をどう読むか').
* ``mfalcon``        3 layers, d=512, 4 heads, 128/128; B=32 histories
                     U{512..4096}; 1024 candidates per user in microbatches of
                     256; score = dot with a 512-d head vector.
* ``full_stack``     8 layers, d=1024, 8 heads, 128/128, B=128, lognormal
                     lengths (median 1000, cap 4096) shortened by Stochastic
                     Length to floor(n^0.8) sampled positions; interleaved
                     content/action tokens from a 1M-id Zipf(1.1) table.

Inputs of the paths around the stack:

* ``full_stack_raw`` / ``raw_stream``  raw (not yet shortened) content/action
                     streams, a 64-bit Stochastic Length seed; tables from
                     ``embedding_table_bits`` (numpy, bf16 bit patterns) or
                     ``device_embedding_table`` (torch's generator on the
                     device, for the 1M x 1024 catalog).
* ``transformer_weights``  the softmax-Transformer comparator layer's weights
                     (dense fp16-rounded, LayerNorm and biases bf16-rounded).

Every array is produced by ``numpy.random.default_rng(seed)`` in a fixed draw
order: lengths -> timestamps -> weights -> rab -> X -> candidates -> head
vector.  bf16 workloads round every bf16-stored tensor to bf16 here (round to
nearest even), so that the float64 oracle and the GPU consume identical
values; rab tables stay fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict
from typing import Dict, List, Optional

import numpy as np

BF16 = "bf16"
FP32 = "fp32"


# ---------------------------------------------------------------------------
# storage rounding (input preparation only)
# ---------------------------------------------------------------------------
def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The uint16 bit patterns of bf16-representable float32 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# descriptors
# ---------------------------------------------------------------------------
@dataclass
class LayerDims:
    d_model: int
    n_heads: int
    d_qk: int
    d_v: int
    n_pos_buckets: int
    n_time_buckets: int
    pos_sub_bits: int
    time_sub_bits: int
    ln_eps: float = 1e-6
    dtype: str = BF16

    @property
    def f1_width(self) -> int:
        return 2 * self.n_heads * self.d_v + 2 * self.n_heads * self.d_qk

    @property
    def hdv(self) -> int:
        return self.n_heads * self.d_v


@dataclass
class Workload:
    name: str
    dims: LayerDims
    n_layers: int
    max_len: int
    offsets: np.ndarray            # int64 [B+1]
    timestamps: np.ndarray         # int64 [T]
    X: np.ndarray                  # float32 [T, d] (bf16-rounded for bf16)
    weights: List[Dict[str, np.ndarray]]
    # M-FALCON only
    cand_offsets: Optional[np.ndarray] = None   # int64 [B+1]
    candidates: Optional[np.ndarray] = None     # float32 [C, d]
    request_ts: Optional[np.ndarray] = None     # int64 [B]
    head_vec: Optional[np.ndarray] = None       # float32 [d]
    microbatch: int = 0
    max_cands: int = 0
    meta: Dict[str, object] = field(default_factory=dict)

    @property
    def B(self) -> int:
        return len(self.offsets) - 1

    @property
    def T(self) -> int:
        return int(self.offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.offsets)


# Sub-bit counts of the log-linear buckets.  Position: the largest S whose
# bucket of (length cap - 1) still fits the table; time: the same for the
# largest 31-bit gap.  These are configuration constants; a CPU test checks
# them against the oracle's bucket function.
POS_SUB_BITS = {"tiny_fp32": 3, "single_layer": 4, "long_history": 3,
                "mfalcon": 3, "full_stack": 4}
TIME_SUB_BITS_BY_BUCKETS = {32: 0, 128: 2}


def _timestamps(rng: np.random.Generator, n: int, mean_gap: float = 60.0) -> np.ndarray:
    """int64 seconds, starting at 0, floor of the running sum of Exp(mean) gaps."""
    gaps = rng.exponential(mean_gap, size=max(n - 1, 0))
    t = np.concatenate([[0.0], np.cumsum(gaps)])
    return np.floor(t).astype(np.int64)


def _xavier(rng: np.random.Generator, fan_out: int, fan_in: int) -> np.ndarray:
    a = math.sqrt(6.0 / (fan_in + fan_out))
    return rng.uniform(-a, a, size=(fan_out, fan_in)).astype(np.float32)


def _layer_weights(rng: np.random.Generator, dims: LayerDims, init: str) -> Dict[str, np.ndarray]:
    d, F, hdv = dims.d_model, dims.f1_width, dims.hdv
    if init == "normal":
        W1 = rng.normal(0.0, 0.02, size=(F, d)).astype(np.float32)
        W2 = rng.normal(0.0, 0.02, size=(d, hdv)).astype(np.float32)
    else:
        W1 = _xavier(rng, F, d)
        W2 = _xavier(rng, d, hdv)
    b1 = rng.normal(0.0, 0.02, size=F).astype(np.float32)
    b2 = rng.normal(0.0, 0.02, size=d).astype(np.float32)
    gamma = (1.0 + rng.normal(0.0, 0.02, size=hdv)).astype(np.float32)
    beta = rng.normal(0.0, 0.02, size=hdv).astype(np.float32)
    return dict(W1=W1, b1=b1, W2=W2, b2=b2, ln_gamma=gamma, ln_beta=beta)


def _rab(rng: np.random.Generator, dims: LayerDims) -> Dict[str, np.ndarray]:
    return dict(
        rab_pos=rng.normal(0.0, 0.02, size=(dims.n_heads, dims.n_pos_buckets)).astype(np.float32),
        rab_time=rng.normal(0.0, 0.02, size=(dims.n_heads, dims.n_time_buckets)).astype(np.float32),
    )


def _finish(w: Workload) -> Workload:
    """Round bf16-stored tensors to bf16 (rab stays fp32)."""
    if w.dims.dtype == BF16:
        w.X = round_to_bf16(w.X)
        for lw in w.weights:
            for k in ("W1", "b1", "W2", "b2", "ln_gamma", "ln_beta"):
                lw[k] = round_to_bf16(lw[k])
        if w.candidates is not None:
            w.candidates = round_to_bf16(w.candidates)
        if w.head_vec is not None:
            w.head_vec = round_to_bf16(w.head_vec)
    return w


def _offsets(lengths: np.ndarray) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def custom(name: str, lengths, dims: LayerDims, n_layers: int = 1, seed: int = 0,
           init: str = "xavier", max_len: Optional[int] = None,
           cands_per_user=None, microbatch: int = 0, x_scale: float = 1.0,
           ts_base=None) -> Workload:
    """A workload with explicit lengths (used by tests for edge cases).

    ``cands_per_user`` (int or list) adds M-FALCON candidates; ``ts_base``
    (list of int64) shifts each user's timestamps by a large epoch.
    """
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    ts = [_timestamps(rng, int(n)) for n in lengths]
    if ts_base is not None:
        ts = [t + np.int64(b) for t, b in zip(ts, ts_base)]
    timestamps = np.concatenate(ts) if B else np.zeros(0, np.int64)
    weights = []
    for _ in range(n_layers):
        lw = _layer_weights(rng, dims, init)
        lw.update(_rab(rng, dims))
        weights.append(lw)
    T = int(lengths.sum())
    X = (x_scale * rng.standard_normal((T, dims.d_model))).astype(np.float32)
    w = Workload(name=name, dims=dims, n_layers=n_layers,
                 max_len=int(max_len if max_len is not None else max(1, int(lengths.max(initial=1)))),
                 offsets=_offsets(lengths), timestamps=timestamps.astype(np.int64),
                 X=X, weights=weights)
    if cands_per_user is not None:
        m = np.broadcast_to(np.asarray(cands_per_user, dtype=np.int64), (B,)).copy()
        C = int(m.sum())
        w.cand_offsets = _offsets(m)
        w.candidates = rng.standard_normal((C, dims.d_model)).astype(np.float32)
        w.request_ts = np.array([t[-1] if len(t) else 0 for t in ts], dtype=np.int64)
        w.head_vec = rng.normal(0.0, 1.0 / math.sqrt(dims.d_model), size=dims.d_model).astype(np.float32)
        w.microbatch = int(microbatch) if microbatch else max(1, int(m.max(initial=1)))
        w.max_cands = int(m.max(initial=0))
    return _finish(w)


# ---------------------------------------------------------------------------
# the five named workloads
# ---------------------------------------------------------------------------
def tiny_fp32(seed: int = 0) -> Workload:
    """1 layer, B=4 users, lengths U{8..64}, d=64, 2 heads, qk/v dim 32; 32 position
    and 32 time-gap log buckets; weights N(0,0.02); X N(0,1); fp32."""
    rng = np.random.default_rng(seed)
    dims = LayerDims(64, 2, 32, 32, 32, 32, POS_SUB_BITS["tiny_fp32"],
                     TIME_SUB_BITS_BY_BUCKETS[32], 1e-6, FP32)
    lengths = rng.integers(8, 65, size=4).astype(np.int64)
    ts = np.concatenate([_timestamps(rng, int(n)) for n in lengths])
    lw = _layer_weights(rng, dims, "normal")
    lw.update(_rab(rng, dims))
    X = rng.standard_normal((int(lengths.sum()), dims.d_model)).astype(np.float32)
    return _finish(Workload("tiny_fp32", dims, 1, 64, _offsets(lengths), ts, X, [lw]))


def _lognormal_lengths(rng, B, median, sigma, lo, hi):
    n = np.round(rng.lognormal(math.log(median), sigma, size=B))
    return np.clip(n, lo, hi).astype(np.int64)


def single_layer(seed: int = 0) -> Workload:
    """1 layer bf16: B=64, lengths lognormal(median 256, sigma 1) capped at 1024,
    d=256, 4 heads, 64/64, 128+128 buckets, Xavier weights, X N(0,1)."""
    rng = np.random.default_rng(seed)
    dims = LayerDims(256, 4, 64, 64, 128, 128, POS_SUB_BITS["single_layer"],
                     TIME_SUB_BITS_BY_BUCKETS[128], 1e-6, BF16)
    lengths = _lognormal_lengths(rng, 64, 256, 1.0, 1, 1024)
    ts = np.concatenate([_timestamps(rng, int(n)) for n in lengths])
    lw = _layer_weights(rng, dims, "xavier")
    lw.update(_rab(rng, dims))
    X = rng.standard_normal((int(lengths.sum()), dims.d_model)).astype(np.float32)
    return _finish(Workload("single_layer", dims, 1, 1024, _offsets(lengths), ts, X, [lw]))


def long_history(seed: int = 0) -> Workload:
    """1 layer bf16: B=16, lengths U{2048..8192}, d=512, 8 heads, head dim 64."""
    rng = np.random.default_rng(seed)
    dims = LayerDims(512, 8, 64, 64, 128, 128, POS_SUB_BITS["long_history"],
                     TIME_SUB_BITS_BY_BUCKETS[128], 1e-6, BF16)
    lengths = rng.integers(2048, 8193, size=16).astype(np.int64)
    ts = np.concatenate([_timestamps(rng, int(n)) for n in lengths])
    lw = _layer_weights(rng, dims, "xavier")
    lw.update(_rab(rng, dims))
    X = rng.standard_normal((int(lengths.sum()), dims.d_model)).astype(np.float32)
    return _finish(Workload("long_history", dims, 1, 8192, _offsets(lengths), ts, X, [lw]))


def mfalcon(seed: int = 0, n_users: int = 32, cands: int = 1024, microbatch: int = 256) -> Workload:
    """M-FALCON ranking: 3-layer stack, d=512, 4 heads, head dim 128; B=32 histories
    U{512..4096}; 1024 N(0,1) candidates per user in microbatches of 256; the
    score is the dot with a 512-d head vector N(0, 1/d)."""
    rng = np.random.default_rng(seed)
    dims = LayerDims(512, 4, 128, 128, 128, 128, POS_SUB_BITS["mfalcon"],
                     TIME_SUB_BITS_BY_BUCKETS[128], 1e-6, BF16)
    lengths = rng.integers(512, 4097, size=n_users).astype(np.int64)
    ts_list = [_timestamps(rng, int(n)) for n in lengths]
    weights = []
    for _ in range(3):
        weights.append(_layer_weights(rng, dims, "xavier"))
    for lw in weights:
        lw.update(_rab(rng, dims))
    X = rng.standard_normal((int(lengths.sum()), dims.d_model)).astype(np.float32)
    m = np.full(n_users, cands, dtype=np.int64)
    candidates = rng.standard_normal((int(m.sum()), dims.d_model)).astype(np.float32)
    head = rng.normal(0.0, 1.0 / math.sqrt(dims.d_model), size=dims.d_model).astype(np.float32)
    w = Workload("mfalcon", dims, 3, 4096, _offsets(lengths), np.concatenate(ts_list), X, weights,
                 cand_offsets=_offsets(m), candidates=candidates,
                 request_ts=np.array([t[-1] for t in ts_list], dtype=np.int64),
                 head_vec=head, microbatch=microbatch, max_cands=cands)
    return _finish(w)


def stochastic_length_keep(n: int) -> int:
    """Stochastic Length keep count: min(n, floor(n**0.8)), at least 1.

    With the 4096 cap this gives 776, the typical shortened length quoted in
    'HSTUとGenerative Recommenders', section '2. Stochastic Lengthで学習時の履歴を間引く'.
    """
    return int(max(1, min(n, math.floor(n ** 0.8))))


def _zipf_cdf(n_ids: int, s: float) -> np.ndarray:
    p = np.arange(1, n_ids + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(p)
    return c / c[-1]


def _embedding_rows(seed: int, table: int, ids: np.ndarray, d: int) -> Dict[int, np.ndarray]:
    """Rows of an N(0,1) embedding table, each drawn from its own (seed, table, id)
    stream, so a row does not depend on which other ids were drawn."""
    out = {}
    for i in np.unique(ids):
        out[int(i)] = np.random.default_rng([seed, 7919, table, int(i)]).standard_normal(d).astype(np.float32)
    return out


def full_stack(seed: int = 0, n_users: int = 128) -> Workload:
    """8-layer stack bf16: d=1024, 8 heads, head dim 128, B=128; raw lengths
    lognormal(median 1000, sigma 1) clipped to [2, 4096], shortened by
    Stochastic Length to floor(n^0.8) random positions (sorted); content and
    action tokens alternate by original position; content ids Zipf(1.1) over
    1M ids (fixed random id permutation), actions uniform over 8 types; token
    embeddings N(0,1); timestamps on the original positions."""
    rng = np.random.default_rng(seed)
    dims = LayerDims(1024, 8, 128, 128, 128, 128, POS_SUB_BITS["full_stack"],
                     TIME_SUB_BITS_BY_BUCKETS[128], 1e-6, BF16)
    raw = _lognormal_lengths(rng, n_users, 1000, 1.0, 2, 4096)
    keep_pos, ts_list = [], []
    for n in raw:
        t_full = _timestamps(rng, int(n))
        k = stochastic_length_keep(int(n))
        pos = np.sort(rng.choice(int(n), size=k, replace=False))
        keep_pos.append(pos)
        ts_list.append(t_full[pos])
    lengths = np.array([len(p) for p in keep_pos], dtype=np.int64)
    weights = []
    for _ in range(8):
        weights.append(_layer_weights(rng, dims, "xavier"))
    for lw in weights:
        lw.update(_rab(rng, dims))
    # token stream: even original positions are content, odd are actions
    n_ids, n_actions = 1_000_000, 8
    cdf = _zipf_cdf(n_ids, 1.1)
    perm = rng.permutation(n_ids)
    kinds, ids = [], []
    for pos in keep_pos:
        is_content = (pos % 2) == 0
        u = rng.random(len(pos))
        rank = np.minimum(np.searchsorted(cdf, u, side="left"), n_ids - 1)
        act = rng.integers(0, n_actions, size=len(pos))
        ids.append(np.where(is_content, perm[rank], act))
        kinds.append(is_content)
    ids_all = np.concatenate(ids)
    kinds_all = np.concatenate(kinds)
    content_rows = _embedding_rows(seed, 0, ids_all[kinds_all], dims.d_model)
    action_rows = _embedding_rows(seed, 1, ids_all[~kinds_all], dims.d_model)
    X = np.empty((len(ids_all), dims.d_model), dtype=np.float32)
    for r, (i, c) in enumerate(zip(ids_all, kinds_all)):
        X[r] = content_rows[int(i)] if c else action_rows[int(i)]
    w = Workload("full_stack", dims, 8, stochastic_length_keep(4096), _offsets(lengths),
                 np.concatenate(ts_list), X, weights,
                 meta=dict(raw_lengths=raw, n_unique_content=len(content_rows)))
    return _finish(w)


@dataclass
class RawStream:
    """Raw (not yet shortened) token streams of a batch of users: the input of
    Stochastic Length + token embedding.  Content and action tokens alternate
    by position (content at even positions); ids index the content table
    (n_content rows) or the action table (n_actions rows)."""
    name: str
    raw_offsets: np.ndarray        # int64 [B+1]
    raw_ids: np.ndarray            # int64 [R]
    raw_timestamps: np.ndarray     # int64 [R]
    n_content: int
    n_actions: int
    d_model: int
    sl_seed: int                   # 64-bit Stochastic Length seed
    max_raw_len: int

    @property
    def B(self) -> int:
        return len(self.raw_offsets) - 1

    @property
    def R(self) -> int:
        return int(self.raw_offsets[-1])


def _raw_stream(rng, name, lengths, d_model, n_content, n_actions, zipf_s, max_raw_len):
    lengths = np.asarray(lengths, np.int64)
    cdf = _zipf_cdf(n_content, zipf_s)
    perm = rng.permutation(n_content)
    ts, ids = [np.zeros(0, np.int64)], [np.zeros(0, np.int64)]
    for n in lengths:
        n = int(n)
        ts.append(_timestamps(rng, n) + int(rng.integers(0, 1 << 31)))
        u = rng.random(n)
        rank = np.minimum(np.searchsorted(cdf, u, side="left"), n_content - 1)
        act = rng.integers(0, n_actions, size=n)
        ids.append(np.where(np.arange(n) % 2 == 0, perm[rank], act).astype(np.int64))
    seed = int(rng.integers(0, 1 << 63)) * 2 + int(rng.integers(0, 2))
    return RawStream(name, _offsets(lengths), np.concatenate(ids), np.concatenate(ts),
                     n_content, n_actions, d_model, seed,
                     int(max_raw_len if max_raw_len is not None else max(lengths.max(initial=0), 1)))


def raw_stream(name: str, lengths, d_model: int, n_content: int, n_actions: int = 8,
               seed: int = 0, zipf_s: float = 1.1, max_raw_len: Optional[int] = None) -> RawStream:
    """Raw streams of the given lengths: per user Exp(60 s) gaps from a random
    31-bit epoch, content ids Zipf(zipf_s) over n_content (fixed random id
    permutation), actions uniform over n_actions, and a random 64-bit seed."""
    return _raw_stream(np.random.default_rng(seed), name, lengths, d_model, n_content, n_actions,
                       zipf_s, max_raw_len)


def full_stack_raw(seed: int = 0, n_users: int = 128) -> RawStream:
    """The raw input of the 8-layer stack workload: B=128 users, raw lengths
    lognormal(median 1000, sigma 1) clipped to [2, 4096], d=1024, content ids
    Zipf(1.1) over 1M ids, 8 action types."""
    rng = np.random.default_rng([seed, 4096])
    raw = _lognormal_lengths(rng, n_users, 1000, 1.0, 2, 4096)
    return _raw_stream(rng, "full_stack_raw", raw, 1024, 1_000_000, 8, 1.1, 4096)


def embedding_table_bits(seed: int, table: int, rows: int, d: int) -> np.ndarray:
    """An N(0,1) embedding table rounded to bf16, as uint16 bit patterns [rows, d]."""
    a = np.random.default_rng([seed, 7919, table]).standard_normal((rows, d), dtype=np.float32)
    return bf16_bits(round_to_bf16(a))


def device_embedding_table(seed: int, table: int, rows: int, d: int, device):
    """An N(0,1) bf16 embedding table [rows, d] drawn by torch's generator on
    `device` (for tables too large to draw on the host; copy it back to feed
    the oracle)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + 7919 * (table + 1)) & ((1 << 63) - 1))
    return torch.randn(rows, d, generator=g, device=device, dtype=torch.bfloat16)


def round_to_f16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest fp16 (ties to even); returns float32."""
    return np.asarray(a, np.float32).astype(np.float16).astype(np.float32)


def transformer_weights(seed: int, d: int, d_ff: int) -> Dict[str, np.ndarray]:
    """Weights of the softmax-Transformer comparator layer: dense weights
    N(0, 1/fan_in) rounded to fp16 (W_qkv [3d, d], W_o [d, d], W_1 [d_ff, d],
    W_2 [d, d_ff]); LayerNorm gamma = 1 + N(0, 0.02), beta and biases
    N(0, 0.02), rounded to bf16."""
    rng = np.random.default_rng([seed, 512, d, d_ff])

    def dense(o, i):
        return round_to_f16(rng.normal(0.0, 1.0 / math.sqrt(i), size=(o, i)).astype(np.float32))

    def small(n, base=0.0):
        return round_to_bf16((base + rng.normal(0.0, 0.02, size=n)).astype(np.float32))
    return dict(ln1_gamma=small(d, 1.0), ln1_beta=small(d), W_qkv=dense(3 * d, d),
                W_o=dense(d, d), ln2_gamma=small(d, 1.0), ln2_beta=small(d), W_1=dense(d_ff, d),
                b_1=small(d_ff), W_2=dense(d, d_ff), b_2=small(d))


WORKLOADS = {
    "tiny_fp32": tiny_fp32,
    "single_layer": single_layer,
    "long_history": long_history,
    "mfalcon": mfalcon,
    "full_stack": full_stack,
}


def make(name: str, seed: int = 0, **kw) -> Workload:
    return WORKLOADS[name](seed=seed, **kw)


def dims_dict(dims: LayerDims) -> dict:
    return asdict(dims)
