"""Seeded synthetic workloads for the HSTU jagged attention path.

This module only draws random numbers and arranges them into the jagged
layouts the library consumes.  It holds none of the method's arithmetic
(no scores, biases, buckets or activations), so the CUDA path and the CPU
oracle can both take their inputs from here without sharing any computation.

Workload shapes follow the five synthetic workloads the HSTU pages motivate:
  * "DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf",
    section "HSTU Hyperparameters" (Table 5: 4 heads, D=512, per-head 128,
    max length 4096, bf16) and section "Model Architecture" (chronological
    item/action/time tokens, candidate appended to the history);
  * the ULTRA-HSTU review (16k histories in production).
Draw order is fixed: lengths, then timestamps, then values, so a seed fixes
every array.  Timestamps are integer seconds: the floor of the running sum of
exponential gaps.  Candidate tokens copy the last history timestamp.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: str                    # "f32" or "bf16"
    num_seqs: int
    len_kind: str                 # "uniform" | "zipf" | "fixed_targets"
    len_lo: int
    len_hi: int
    num_heads: int
    d_qk: int
    d_v: int
    gap_mean_s: float
    pos_lo: int
    pos_hi: int
    num_time_buckets: int
    n_scale: int                  # the N in the 1/N scale
    d_model: Optional[int] = None  # layer workloads only
    num_layers: int = 1
    num_targets: int = 0          # candidates appended to each history
    zipf_a: float = 1.2
    value_std: float = 1.0        # Q/K/V (attention) or X (layer) std
    weight_std: float = 0.02
    table_std: float = 0.1
    has_bwd: bool = False

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def is_layer(self) -> bool:
        return self.d_model is not None


WORKLOADS = {
    w.name: w
    for w in [
        # Single small fp32 layer, forward only.
        Workload("layer_f32_small", 0, "f32", 4, "uniform", 16, 128, 2, 32, 32,
                 60.0, 0, 127, 32, 128, d_model=64, value_std=1.0),
        # Short-history bf16 attention, forward and backward.
        Workload("attn_bf16_short", 1, "bf16", 32, "uniform", 64, 1024, 4, 64, 64,
                 300.0, -1024, 1024, 64, 1024, has_bwd=True),
        # Eight-layer bf16 stack forward over Zipf-length histories.
        Workload("layer_stack_bf16", 2, "bf16", 64, "zipf", 32, 4096, 4, 128, 128,
                 300.0, -4096, 4096, 128, 4096, d_model=512, num_layers=8,
                 value_std=0.02),
        # Ranking inference: 2048 history tokens + 512 candidates per user.
        Workload("ranking_bf16", 3, "bf16", 16, "fixed_targets", 2560, 2560, 2, 128, 128,
                 120.0, -2560, 2560, 128, 2560, d_model=256, num_targets=512,
                 value_std=0.02),
        # Long-history training step: forward + backward with bias-table grads.
        Workload("long_history_bf16", 4, "bf16", 8, "uniform", 8192, 16384, 4, 128, 128,
                 300.0, -4096, 4096, 128, 16384, has_bwd=True),
    ]
}

BY_INDEX = {w.index: w for w in WORKLOADS.values()}


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def draw_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.len_kind == "uniform":
        return rng.integers(w.len_lo, w.len_hi + 1, size=w.num_seqs).astype(np.int64)
    if w.len_kind == "zipf":
        return np.clip(rng.zipf(w.zipf_a, size=w.num_seqs), w.len_lo, w.len_hi).astype(np.int64)
    if w.len_kind == "fixed_targets":
        return np.full(w.num_seqs, w.len_lo, dtype=np.int64)
    raise ValueError(w.len_kind)


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def draw_timestamps(rng: np.random.Generator, lengths, gap_mean_s: float,
                    num_targets=None, epoch: int = 0) -> np.ndarray:
    """int64 seconds, non-decreasing within each sequence.

    History token k of a sequence is stamped floor(sum of the first k+1
    exponential gaps); candidate tokens copy the last history stamp.
    """
    out = []
    for b, L in enumerate(lengths):
        L = int(L)
        nt = 0 if num_targets is None else int(num_targets[b])
        nh = L - nt
        gaps = rng.exponential(gap_mean_s, size=nh)
        t = np.floor(np.cumsum(gaps)).astype(np.int64) + epoch
        if nt:
            last = t[-1] if nh else np.int64(epoch)
            t = np.concatenate([t, np.full(nt, last, dtype=np.int64)])
        out.append(t)
    if not out:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate(out).astype(np.int64)


def _normal(rng, shape, std, dtype):
    a = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return torch.from_numpy(a).to(dtype)


@dataclasses.dataclass
class AttnInputs:
    seq_offsets: torch.Tensor   # int64 [B+1]
    timestamps: torch.Tensor    # int64 [T]
    num_targets: Optional[torch.Tensor]  # int32 [B] or None
    q: torch.Tensor             # [T, h, d_qk]
    k: torch.Tensor
    v: torch.Tensor             # [T, h, d_v]
    rab_pos: torch.Tensor       # f32 [pos_hi - pos_lo + 1]
    rab_time: torch.Tensor      # f32 [num_time_buckets]
    dout: Optional[torch.Tensor]  # [T, h, d_v] (backward workloads)
    pos_lo: int
    pos_hi: int
    inv_n: float
    max_seq_len: int

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets.numpy())


@dataclasses.dataclass
class LayerWeights:
    w1: torch.Tensor      # [D, h*(2 d_v + 2 d_qk)]
    b1: torch.Tensor      # [h*(2 d_v + 2 d_qk)]
    w2: torch.Tensor      # [h*d_v, D]
    b2: torch.Tensor      # [D]
    ln_gamma: torch.Tensor  # f32 [h*d_v]
    ln_beta: torch.Tensor   # f32 [h*d_v]


@dataclasses.dataclass
class LayerInputs:
    x: torch.Tensor                 # [T, D]
    layers: List[LayerWeights]
    attn: AttnInputs                # q/k/v are None-like placeholders (unused)


def make_attn_inputs(rng: np.random.Generator, lengths, num_heads: int, d_qk: int, d_v: int,
                     gap_mean_s: float, pos_lo: int, pos_hi: int, num_time_buckets: int,
                     n_scale: float, dtype: torch.dtype, value_std: float = 1.0,
                     table_std: float = 0.1, num_targets=None, with_dout: bool = False,
                     epoch: int = 0, with_values: bool = True) -> AttnInputs:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = draw_timestamps(rng, lengths, gap_mean_s, num_targets, epoch=epoch)
    if with_values:
        q = _normal(rng, (T, num_heads, d_qk), value_std, dtype)
        k = _normal(rng, (T, num_heads, d_qk), value_std, dtype)
        v = _normal(rng, (T, num_heads, d_v), value_std, dtype)
    else:
        q = k = v = None
    rab_pos = _normal(rng, (pos_hi - pos_lo + 1,), table_std, torch.float32)
    rab_time = _normal(rng, (num_time_buckets,), table_std, torch.float32)
    dout = _normal(rng, (T, num_heads, d_v), 1.0, dtype) if with_dout else None
    nt = None if num_targets is None else torch.from_numpy(np.asarray(num_targets, dtype=np.int32))
    return AttnInputs(torch.from_numpy(off), torch.from_numpy(ts), nt, q, k, v, rab_pos, rab_time,
                      dout, pos_lo, pos_hi, 1.0 / float(n_scale),
                      int(lengths.max()) if len(lengths) else 0)


def make_layer_weights(rng: np.random.Generator, d_model: int, num_heads: int, d_qk: int, d_v: int,
                       dtype: torch.dtype, weight_std: float = 0.02, random_affine: bool = False):
    width = num_heads * (2 * d_v + 2 * d_qk)
    w1 = _normal(rng, (d_model, width), weight_std, dtype)
    w2 = _normal(rng, (num_heads * d_v, d_model), weight_std, dtype)
    if random_affine:
        b1 = _normal(rng, (width,), 0.05, dtype)
        b2 = _normal(rng, (d_model,), 0.05, dtype)
        g = 1.0 + _normal(rng, (num_heads * d_v,), 0.1, torch.float32)
        be = _normal(rng, (num_heads * d_v,), 0.1, torch.float32)
    else:
        b1 = torch.zeros(width, dtype=dtype)
        b2 = torch.zeros(d_model, dtype=dtype)
        g = torch.ones(num_heads * d_v, dtype=torch.float32)
        be = torch.zeros(num_heads * d_v, dtype=torch.float32)
    return LayerWeights(w1, b1, w2, b2, g, be)


def generate(w: Workload, seed: Optional[int] = None, num_seqs: Optional[int] = None,
             len_hi: Optional[int] = None):
    """Build the seeded inputs of workload `w`.

    `num_seqs` / `len_hi` shrink the workload (for oracle-sized tests) while
    keeping its distributions; the seed still fixes every draw.
    """
    rng = np.random.default_rng(w.seed if seed is None else seed)
    if num_seqs is not None or len_hi is not None:
        w = dataclasses.replace(w, num_seqs=num_seqs or w.num_seqs,
                                len_hi=min(len_hi or w.len_hi, w.len_hi),
                                len_lo=min(w.len_lo, len_hi or w.len_hi))
    lengths = draw_lengths(w, rng)
    nt = None
    if w.num_targets:
        ntv = min(w.num_targets, int(lengths.min()) // 2) if len_hi else w.num_targets
        nt = np.full(w.num_seqs, ntv, dtype=np.int32)
    dt = torch_dtype(w)
    if not w.is_layer:
        return make_attn_inputs(rng, lengths, w.num_heads, w.d_qk, w.d_v, w.gap_mean_s,
                                w.pos_lo, w.pos_hi, w.num_time_buckets, w.n_scale, dt,
                                value_std=w.value_std, table_std=w.table_std,
                                num_targets=nt, with_dout=w.has_bwd)
    attn = make_attn_inputs(rng, lengths, w.num_heads, w.d_qk, w.d_v, w.gap_mean_s,
                            w.pos_lo, w.pos_hi, w.num_time_buckets, w.n_scale, dt,
                            table_std=w.table_std, num_targets=nt, with_values=False)
    T = attn.total_tokens
    x = _normal(rng, (T, w.d_model), w.value_std, dt)
    layers = [make_layer_weights(rng, w.d_model, w.num_heads, w.d_qk, w.d_v, dt, w.weight_std)
              for _ in range(w.num_layers)]
    return LayerInputs(x, layers, attn)
