"""Data parallelism for the jagged attention step: one process per GPU.

Sequences are independent (each user history is its own causal block, the
DLRMv4 page's "Model Architecture" section), so a global batch is split by
sequence across ranks and the forward needs no exchange.  The backward's only
shared parameters are the two relative-bias tables: their gradients are
summed across ranks with one all-reduce of pos+time floats.

`lpt_partition` balances ranks by the attention cost of each sequence
(~ visible pairs, quadratic in length), longest first, the same goal as the
load balancing the ULTRA-HSTU review describes for stochastic-length
training.
"""

from __future__ import annotations

import dataclasses
from typing import List, Sequence

import numpy as np
import torch

from . import flops


def sequence_costs(lengths: Sequence[int], num_targets=None) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    nts = np.zeros_like(lengths) if num_targets is None else np.asarray(num_targets, dtype=np.int64)
    return np.array([flops.attn_pairs_per_seq(L, n) for L, n in zip(lengths, nts)], dtype=np.int64)


def lpt_partition(costs: Sequence[int], world: int) -> List[List[int]]:
    """Greedy longest-processing-time assignment of items to `world` bins.

    Deterministic: items in order of decreasing cost (ties by index), each to
    the currently lightest bin (ties by rank).  Each bin's indices are
    returned in increasing order.
    """
    costs = np.asarray(costs, dtype=np.int64)
    order = sorted(range(len(costs)), key=lambda i: (-int(costs[i]), i))
    load = [0] * world
    bins: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        bins[r].append(i)
        load[r] += int(costs[i])
    return [sorted(b) for b in bins]


def dp_shard_inputs(w, world: int, rank: int):
    """This rank's share of a global batch of `world` x `w.num_seqs` sequences of
    workload `w` (a `workloads.Workload` without layers), for weak scaling: the
    global lengths come from the workload's seed, `lpt_partition` assigns whole
    sequences to ranks by cost, and the rank draws its own sequences' values from
    its own seed.  The bias tables, parameters shared by every rank, come from
    one seed, so all ranks hold the same tables."""
    from . import workloads
    gw = dataclasses.replace(w, num_seqs=w.num_seqs * world)
    lengths = workloads.draw_lengths(gw, np.random.default_rng(w.seed))
    mine = lengths[lpt_partition(sequence_costs(lengths), world)[rank]]
    dt = workloads.torch_dtype(w)
    inp = workloads.make_attn_inputs(np.random.default_rng(w.seed + 1 + rank), mine, w.num_heads, w.d_qk, w.d_v,
                                     w.gap_mean_s, w.pos_lo, w.pos_hi, w.num_time_buckets, w.n_scale, dt,
                                     value_std=w.value_std, table_std=w.table_std, with_dout=w.has_bwd)
    tables = workloads.make_attn_inputs(np.random.default_rng(w.seed), [1], w.num_heads, w.d_qk, w.d_v,
                                        w.gap_mean_s, w.pos_lo, w.pos_hi, w.num_time_buckets, w.n_scale, dt,
                                        table_std=w.table_std, with_values=False)
    return dataclasses.replace(inp, rab_pos=tables.rab_pos, rab_time=tables.rab_time)


def shard_attn_inputs(inp, seqs: Sequence[int]):
    """The sequences `seqs` of a `workloads.AttnInputs` as a new jagged batch."""
    off = inp.seq_offsets.numpy()
    sl = [slice(int(off[b]), int(off[b + 1])) for b in seqs]
    lengths = [s.stop - s.start for s in sl]
    new_off = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))

    def cat(t):
        if t is None:
            return None
        if not sl:
            return t[:0].clone()
        return torch.cat([t[s] for s in sl])

    nt = None if inp.num_targets is None else inp.num_targets[list(seqs)].clone()
    return dataclasses.replace(inp, seq_offsets=new_off, timestamps=cat(inp.timestamps),
                               num_targets=nt, q=cat(inp.q), k=cat(inp.k), v=cat(inp.v),
                               dout=cat(inp.dout), max_seq_len=max(lengths) if lengths else 0)


def allreduce_bias_grads(d_rab_pos: torch.Tensor, d_rab_time: torch.Tensor, group=None) -> None:
    """Sum both bias-table gradients over all ranks in place (one collective)."""
    import torch.distributed as dist

    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    npos = d_rab_pos.numel()
    if d_rab_pos.data_ptr() + 4 * npos == d_rab_time.data_ptr() and d_rab_pos.is_contiguous():
        # the two tables are adjacent views of one buffer: reduce it in one call
        flat = torch.as_strided(d_rab_pos, (npos + d_rab_time.numel(),), (1,))
        dist.all_reduce(flat, group=group)
        return
    flat = torch.cat([d_rab_pos.reshape(-1), d_rab_time.reshape(-1)])
    dist.all_reduce(flat, group=group)
    d_rab_pos.copy_(flat[:npos].view_as(d_rab_pos))
    d_rab_time.copy_(flat[npos:].view_as(d_rab_time))


# parameter gradients of one transduction layer (per-token dx stays on its rank)
LAYER_PARAM_GRADS = ("dw1", "db1", "dw2", "db2", "d_ln_gamma", "d_ln_beta", "d_rab_pos", "d_rab_time")


def allreduce_layer_grads(grads: dict, group=None) -> None:
    """Sum a layer's parameter gradients (the dict of `ops.hstu_layer_bwd`) over
    all ranks in place, packed into one buffer and one all-reduce."""
    import torch.distributed as dist

    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    parts = [grads[k] for k in LAYER_PARAM_GRADS]
    flat = torch.cat([t.reshape(-1) for t in parts])
    dist.all_reduce(flat, group=group)
    o = 0
    for t in parts:
        n = t.numel()
        t.copy_(flat[o:o + n].view_as(t))
        o += n
