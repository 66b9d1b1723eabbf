"""GPU parity of the two bias options the pages leave open, against the oracle
under the same reading (through the C ABI):

- candidates at their own index (cand_own_index): candidate i sits at position i
  instead of the first position after the history ("DLRMv4 Brings
  Sequence-Based Recommendation Training to MLPerf", "Model Architecture", gives
  positions only for the history);
- one pair of bias tables per head (rab_pos [H, entries], rab_time [H, NB])
  instead of one pair shared by the heads.

Every case first checks that the oracle's answer under the other reading is far
outside the tolerance, so that a kernel which ignored the option would fail."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import (assert_bf16_close, assert_f32_close, gpu_bwd, gpu_fwd, maxabs_rel_err, to_dev)

pytestmark = pytest.mark.gpu

NAMES = ["dq", "dk", "dv", "d_rab_pos", "d_rab_time"]


def _inputs(lengths, nt, H, d, dtype, seed, per_head, lo=-300, hi=300, nb=32, gap=300.0):
    # small q, k and unit-scale tables: the bias carries a large share of every score
    rng = np.random.default_rng(seed)
    inp = workloads.make_attn_inputs(rng, lengths, H, d, d, gap, lo, hi, nb, max(lengths), dtype,
                                     value_std=0.35, table_std=1.0, num_targets=nt, with_dout=True)
    if per_head:
        t = np.random.default_rng(seed + 1000)
        rp = torch.from_numpy(t.standard_normal((H, hi - lo + 1)).astype(np.float32))
        rt = torch.from_numpy(t.standard_normal((H, nb)).astype(np.float32))
        inp = dataclasses.replace(inp, rab_pos=rp, rab_time=rt)
    return inp


def _args(inp):
    return (inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v, inp.rab_pos, inp.rab_time,
            inp.pos_lo, inp.pos_hi, inp.inv_n)


def _shared(inp):
    """The same inputs with every head reading head 0's tables."""
    if inp.rab_pos.dim() == 1:
        return inp
    H = inp.rab_pos.shape[0]
    return dataclasses.replace(inp, rab_pos=inp.rab_pos[:1].expand(H, -1).contiguous(),
                               rab_time=inp.rab_time[:1].expand(H, -1).contiguous())


def _assert_discriminates(inp, own, ref_out, tol, **win):
    """The other reading of each option set moves the output well past tol."""
    others = []
    if own:
        others.append(oracle.attn_fwd(*_args(inp), cand_own_index=False, **win))
    if inp.rab_pos.dim() == 2:
        others.append(oracle.attn_fwd(*_args(_shared(inp)), cand_own_index=own, **win))
    for o in others:
        assert maxabs_rel_err(o, ref_out) > 5 * tol, "the case does not tell the readings apart"


CASES = [(own, ph) for own in (False, True) for ph in (False, True) if own or ph]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("own,per_head", CASES)
def test_readings_fwd_bwd_bf16(cuda_device, d, own, per_head):
    # ragged: several tiles, ragged tails, an empty and a one-token sequence, a
    # candidate block crossing a tile edge, all-candidate sequences
    lengths = [1, 0, 63, 64, 65, 200, 129, 300]
    nt = [0, 0, 5, 64, 64, 17, 1, 150]
    inp = _inputs(lengths, nt, 2, d, torch.bfloat16, 40 + d, per_head)
    ref = oracle.attn_fwd(*_args(inp), cand_own_index=own)
    _assert_discriminates(inp, own, ref, 2e-2)
    assert_bf16_close(gpu_fwd(inp, cuda_device, cand_own_index=own), ref, what=f"fwd own={own} ph={per_head}")
    g = gpu_bwd(inp, cuda_device, cand_own_index=own)
    r = oracle.attn_bwd(*_args(inp), inp.dout, cand_own_index=own)
    assert tuple(g[3].shape) == tuple(inp.rab_pos.shape) and tuple(g[4].shape) == tuple(inp.rab_time.shape)
    for n, a, b in zip(NAMES, g, r):
        assert_bf16_close(a, b, what=f"bwd own={own} ph={per_head} {n}")


@pytest.mark.parametrize("own,per_head", CASES)
def test_readings_fwd_bwd_f32(cuda_device, own, per_head):
    inp = _inputs([1, 70, 128, 33, 90], [0, 3, 0, 2, 40], 2, 32, torch.float32, 7, per_head, lo=0, hi=127,
                  gap=60.0)
    ref = oracle.attn_fwd(*_args(inp), cand_own_index=own)
    _assert_discriminates(inp, own, ref, 1e-4)
    assert_f32_close(gpu_fwd(inp, cuda_device, cand_own_index=own), ref, what="fwd f32")
    g = gpu_bwd(inp, cuda_device, cand_own_index=own)
    r = oracle.attn_bwd(*_args(inp), inp.dout, cand_own_index=own)
    for n, a, b in zip(NAMES, g, r):
        assert_f32_close(a, b, what=f"bwd f32 {n}")


@pytest.mark.parametrize("d", [64, 128])
def test_readings_with_semi_local_window(cuda_device, d):
    # the window measures distances on the same axis: with own-index candidates a
    # candidate far past the history loses the history keys beyond the window
    win = dict(local_window=40, global_window=8)
    inp = _inputs([260, 1, 97, 150], [60, 0, 30, 150], 2, d, torch.bfloat16, 90 + d, True)
    ref = oracle.attn_fwd(*_args(inp), cand_own_index=True, **win)
    _assert_discriminates(inp, True, ref, 2e-2, **win)
    assert_bf16_close(gpu_fwd(inp, cuda_device, cand_own_index=True, **win), ref, what="fwd window")
    g = gpu_bwd(inp, cuda_device, cand_own_index=True, **win)
    r = oracle.attn_bwd(*_args(inp), inp.dout, cand_own_index=True, **win)
    for n, a, b in zip(NAMES, g, r):
        assert_bf16_close(a, b, what=f"bwd window {n}")


def test_readings_ranking_shapes(cuda_device):
    # the ranking shapes (2,048 history + 512 candidates per user, d = 128) at two
    # users, both options on
    inp = _inputs([2560, 2560], [512, 512], 2, 128, torch.bfloat16, 5, True, lo=-2560, hi=2560, nb=128,
                  gap=120.0)
    ref = oracle.attn_fwd(*_args(inp), cand_own_index=True)
    _assert_discriminates(inp, True, ref, 2e-2)
    assert_bf16_close(gpu_fwd(inp, cuda_device, cand_own_index=True), ref, what="ranking fwd")


def test_readings_layer_fwd_bwd(cuda_device):
    # one transduction layer with per-head tables and own-index candidates
    H, d, D = 2, 64, 128
    rng = np.random.default_rng(77)
    inp = _inputs([100, 1, 37, 0, 98], [10, 0, 0, 0, 30], H, d, torch.bfloat16, 77, True, lo=-200, hi=200)
    lw = workloads.make_layer_weights(rng, D, H, d, d, torch.bfloat16, weight_std=0.1, random_affine=True)
    T = inp.total_tokens
    x = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(torch.bfloat16)
    dev = cuda_device
    kw = dict(num_heads=H, d_qk=d, d_v=d, max_seq_len=inp.max_seq_len, inv_n=inp.inv_n, pos_lo=inp.pos_lo,
              pos_hi=inp.pos_hi, cand_own_index=True)
    xd = to_dev(x, dev)
    prm = [to_dev(t, dev) for t in (lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta)]
    seq = [to_dev(t, dev) for t in (inp.seq_offsets, inp.timestamps, inp.num_targets, inp.rab_pos, inp.rab_time)]
    uvqk = torch.empty((T, H * 4 * d), dtype=torch.bfloat16, device=dev)
    o = torch.empty((T, H * d), dtype=torch.bfloat16, device=dev)
    y = ops.hstu_layer_fwd(xd, *prm, *seq, saved_uvqk=uvqk, saved_o=o, **kw)
    w1, b1, w2, _, g, be = prm
    grads = ops.hstu_layer_bwd(xd, w1, b1, w2, g, be, *seq, uvqk, o, to_dev(dy, dev), **kw)
    torch.cuda.synchronize()
    okw = dict(cand_own_index=True)
    ry, _, ro = oracle.layer_fwd(inp.seq_offsets, inp.timestamps, inp.num_targets, x, lw.w1, lw.b1, lw.w2, lw.b2,
                                 lw.ln_gamma, lw.ln_beta, inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi,
                                 inp.inv_n, H, d, d, want_intermediates=True, **okw)
    assert_bf16_close(o, ro, what="layer attention output")
    assert_bf16_close(y, ry, what="layer output")
    ref = oracle.layer_bwd(inp.seq_offsets, inp.timestamps, inp.num_targets, x, lw.w1, lw.b1, lw.w2,
                           lw.ln_gamma, lw.ln_beta, inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n,
                           H, d, d, dy, **okw)
    for n in ["dx", "dw1", "db1", "dw2", "db2", "d_ln_gamma", "d_ln_beta", "d_rab_pos", "d_rab_time"]:
        assert_bf16_close(grads[n], ref[n], what=f"layer {n}")
    assert tuple(grads["d_rab_pos"].shape) == (H, inp.pos_hi - inp.pos_lo + 1)
