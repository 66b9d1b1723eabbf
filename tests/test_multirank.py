"""Data-parallel host logic on CPU ranks (gloo, world size 2).

Each rank takes its LPT shard of a small jagged batch, runs the oracle
backward on it, and sums the bias-table gradients with the same all-reduce
the GPU step uses; the result must equal the oracle on the whole batch."""

import dataclasses
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


def _batch(per_head=False):
    rng = np.random.default_rng(31)
    inp = workloads.make_attn_inputs(rng, [9, 3, 14, 1, 7, 0, 12], 2, 4, 4, 30.0, -6, 6, 5, 16,
                                     torch.float32, num_targets=[2, 0, 3, 0, 0, 0, 1],
                                     with_dout=True)
    if per_head:  # one table pair per head: the all-reduce keeps the [H, entries] shapes
        inp = dataclasses.replace(inp, rab_pos=torch.stack([inp.rab_pos, 0.5 - inp.rab_pos]),
                                  rab_time=torch.stack([inp.rab_time, 2.0 * inp.rab_time]))
    return inp


def _worker(rank, world, port, out_dir, per_head=False, own=False):
    import torch.distributed as dist

    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _batch(per_head)
        costs = parallel.sequence_costs(inp.lengths, inp.num_targets.numpy())
        mine = parallel.lpt_partition(costs, world)[rank]
        sh = parallel.shard_attn_inputs(inp, mine)
        if sh.total_tokens:
            dq, dk, dv, drp, drt = oracle.attn_bwd(sh.seq_offsets, sh.timestamps, sh.num_targets, sh.q,
                                                   sh.k, sh.v, sh.rab_pos, sh.rab_time, sh.pos_lo,
                                                   sh.pos_hi, sh.inv_n, sh.dout, threads=1, cand_own_index=own)
        else:
            dq = dk = dv = np.zeros((0,))
            drp, drt = np.zeros(tuple(inp.rab_pos.shape)), np.zeros(tuple(inp.rab_time.shape))
        gp, gt = torch.from_numpy(drp.copy()), torch.from_numpy(drt.copy())
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


def test_dp_shards_of_a_global_batch():
    # the multi-GPU bench's inputs: every global sequence on exactly one rank,
    # ranks balanced by visible pairs, one set of bias tables for all
    w = workloads.WORKLOADS["attn_bf16_short"]
    world = 4
    gw = dataclasses.replace(w, num_seqs=w.num_seqs * world)
    glob = workloads.draw_lengths(gw, np.random.default_rng(w.seed))
    shards = [parallel.dp_shard_inputs(w, world, r) for r in range(world)]
    assert sorted(sum((list(s.lengths) for s in shards), [])) == sorted(glob.tolist())
    loads = [int(parallel.sequence_costs(s.lengths).sum()) for s in shards]
    assert max(loads) - min(loads) <= int(parallel.sequence_costs(glob).max())
    for s in shards:
        assert torch.equal(s.rab_pos, shards[0].rab_pos) and torch.equal(s.rab_time, shards[0].rab_time)
        assert s.inv_n == shards[0].inv_n and s.q.shape[0] == s.total_tokens


def test_sequence_costs_are_visible_pairs():
    assert list(parallel.sequence_costs([4, 5], [0, 2])) == [10, 6 + 2 * 4]


@pytest.mark.parametrize("per_head,own", [(False, False), (True, True)])
def test_dp_shards_reproduce_full_batch_gradients(tmp_path, per_head, own):
    import oracle
    oracle.build()
    world = 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path), per_head, own), nprocs=world, join=True,
                       start_method="spawn")
    inp = _batch(per_head)
    full = oracle.attn_bwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                           inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, inp.dout,
                           threads=1, cand_own_index=own)
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


def _layer_batch():
    rng = np.random.default_rng(41)
    attn = workloads.make_attn_inputs(rng, [8, 2, 11, 0, 6, 13], 2, 4, 4, 30.0, -6, 6, 5, 16, torch.float32,
                                      num_targets=[1, 0, 2, 0, 0, 3], with_values=False)
    T, D, W, hv = attn.total_tokens, 6, 2 * 4 * 4, 8
    prm = {"x": rng.standard_normal((T, D)), "w1": rng.standard_normal((D, W)) * 0.4,
           "b1": rng.standard_normal(W) * 0.1, "w2": rng.standard_normal((hv, D)),
           "g": 1 + 0.1 * rng.standard_normal(hv), "be": 0.1 * rng.standard_normal(hv),
           "dy": rng.standard_normal((T, D))}
    return attn, prm


def _layer_grads(attn, prm, rows=None, off=None, nt=None):
    import oracle
    x, dy, ts = prm["x"], prm["dy"], attn.timestamps.numpy()
    if rows is not None:
        x, dy, ts = x[rows], dy[rows], ts[rows]
    return oracle.layer_bwd(attn.seq_offsets if off is None else off, ts,
                            attn.num_targets if nt is None else nt, x, prm["w1"], prm["b1"], prm["w2"],
                            prm["g"], prm["be"], attn.rab_pos, attn.rab_time, attn.pos_lo, attn.pos_hi,
                            attn.inv_n, 2, 4, 4, dy, threads=1)


def _layer_worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        attn, prm = _layer_batch()
        costs = parallel.sequence_costs(attn.lengths, attn.num_targets.numpy())
        mine = parallel.lpt_partition(costs, world)[rank]
        off = attn.seq_offsets.numpy()
        rows = np.concatenate([np.arange(off[b], off[b + 1]) for b in mine]).astype(np.int64)
        sub_off = np.concatenate([[0], np.cumsum([off[b + 1] - off[b] for b in mine])]).astype(np.int64)
        g = _layer_grads(attn, prm, rows, sub_off, attn.num_targets[list(mine)])
        grads = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in g.items()}
        parallel.allreduce_layer_grads(grads)
        np.savez(os.path.join(out_dir, f"layer{rank}.npz"), rows=rows, **{k: v.numpy() for k, v in grads.items()})
    finally:
        dist.destroy_process_group()


def test_dp_layer_backward_sums_parameter_gradients(tmp_path):
    import oracle
    oracle.build()
    world = 2
    port = _free_port()
    mp.start_processes(_layer_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    attn, prm = _layer_batch()
    full = _layer_grads(attn, prm)
    seen = []
    for rank in range(world):
        z = np.load(tmp_path / f"layer{rank}.npz")
        for k in parallel.LAYER_PARAM_GRADS:
            np.testing.assert_allclose(z[k], full[k], rtol=1e-12, atol=1e-12, err_msg=k)
        np.testing.assert_allclose(z["dx"], full["dx"][z["rows"]], rtol=1e-12, atol=1e-12)
        seen += list(z["rows"])
    assert sorted(seen) == list(range(attn.total_tokens))
