"""Data-parallel host logic on CPU ranks (gloo, world size 2).

Each rank takes its LPT shard of a small jagged batch, runs the oracle
backward on it, and sums the bias-table gradients with the same all-reduce
the GPU step uses; the result must equal the oracle on the whole batch."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from hstu_sequential_transduction_b200 import parallel, workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    rng = np.random.default_rng(31)
    return workloads.make_attn_inputs(rng, [9, 3, 14, 1, 7, 0, 12], 2, 4, 4, 30.0, -6, 6, 5, 16,
                                      torch.float32, num_targets=[2, 0, 3, 0, 0, 0, 1],
                                      with_dout=True)


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _batch()
        costs = parallel.sequence_costs(inp.lengths, inp.num_targets.numpy())
        mine = parallel.lpt_partition(costs, world)[rank]
        sh = parallel.shard_attn_inputs(inp, mine)
        if sh.total_tokens:
            dq, dk, dv, drp, drt = oracle.attn_bwd(sh.seq_offsets, sh.timestamps, sh.num_targets, sh.q,
                                                   sh.k, sh.v, sh.rab_pos, sh.rab_time, sh.pos_lo,
                                                   sh.pos_hi, sh.inv_n, sh.dout, threads=1)
        else:
            dq = dk = dv = np.zeros((0,))
            drp, drt = np.zeros(inp.rab_pos.numel()), np.zeros(inp.rab_time.numel())
        buf = torch.from_numpy(np.concatenate([drp, drt]))
        gp, gt = buf[:drp.size], buf[drp.size:]
        parallel.allreduce_bias_grads(gp, gt)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), seqs=np.array(mine), dq=dq, dk=dk, dv=dv,
                 drp=gp.numpy(), drt=gt.numpy())
    finally:
        dist.destroy_process_group()


def test_lpt_partition_balances_and_is_deterministic():
    costs = [100, 1, 50, 50, 7, 0, 99]
    a = parallel.lpt_partition(costs, 2)
    assert a == parallel.lpt_partition(costs, 2)
    assert sorted(sum(a, [])) == list(range(len(costs)))
    loads = [sum(costs[i] for i in b) for b in a]
    assert max(loads) - min(loads) <= max(costs)
    assert parallel.lpt_partition(costs, 1) == [list(range(len(costs)))]
    assert parallel.lpt_partition([], 3) == [[], [], []]


def test_sequence_costs_are_visible_pairs():
    assert list(parallel.sequence_costs([4, 5], [0, 2])) == [10, 6 + 2 * 4]


def test_dp_shards_reproduce_full_batch_gradients(tmp_path):
    import oracle
    oracle.build()
    world = 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    inp = _batch()
    full = oracle.attn_bwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                           inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, inp.dout,
                           threads=1)
    off = inp.seq_offsets.numpy()
    covered = []
    for rank in range(world):
        z = np.load(tmp_path / f"rank{rank}.npz")
        np.testing.assert_allclose(z["drp"], full[3], rtol=0, atol=1e-12)
        np.testing.assert_allclose(z["drt"], full[4], rtol=0, atol=1e-12)
        rows = np.concatenate([np.arange(off[b], off[b + 1]) for b in z["seqs"]]) if len(z["seqs"]) else []
        if len(rows):
            np.testing.assert_allclose(z["dq"], full[0][rows], rtol=0, atol=1e-12)
            np.testing.assert_allclose(z["dv"], full[2][rows], rtol=0, atol=1e-12)
        covered += list(z["seqs"])
    assert sorted(covered) == list(range(len(off) - 1))
