"""GPU parity of the attention-truncation gather (hstu_jagged_truncate) against
the oracle: the kept rows and offsets must be bit-exact, and layers run on the
kept batch must match the oracle's layers on the oracle's kept batch."""

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, rows_of, to_dev

pytestmark = pytest.mark.gpu


def _offsets(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def _check_exact(off, nt, keep, rows, dev):
    new_off, kept = ops.hstu_jagged_truncate(to_dev(torch.from_numpy(off), dev),
                                             None if nt is None else to_dev(torch.from_numpy(nt), dev),
                                             keep, rows.to(dev))
    torch.cuda.synchronize()
    ref_off, ref_rows = oracle.jagged_truncate(off, nt, keep, rows.cpu().numpy() if rows.dtype != torch.bfloat16
                                               else rows.cpu().view(torch.int16).numpy())
    got_off = new_off.cpu().numpy()
    np.testing.assert_array_equal(got_off, ref_off)
    n = int(got_off[-1])
    got = kept[:n].cpu()
    got = got.view(torch.int16).numpy() if got.dtype == torch.bfloat16 else got.numpy()
    np.testing.assert_array_equal(got, ref_rows)
    return got_off


def test_truncate_hand_batch(cuda_device):
    off = np.array([0, 5, 5, 7, 11], np.int64)
    nt = np.array([1, 0, 0, 2], np.int32)
    rows = torch.arange(11, dtype=torch.float32)
    expect = {2: [0, 3, 3, 5, 9], 1: [0, 2, 2, 3, 6], 0: [0, 1, 1, 1, 3]}
    for keep, e in expect.items():
        assert _check_exact(off, nt, keep, rows, cuda_device).tolist() == e


@pytest.mark.parametrize("shape,dtype", [((), torch.int64), ((512,), torch.bfloat16), ((6,), torch.bfloat16),
                                         ((3,), torch.float32), ((4, 8), torch.float32)])
def test_truncate_ragged_row_kinds(cuda_device, shape, dtype):
    """Rows of 8, 1024, 12, 12 and 128 bytes (16-byte and 4-byte copy paths);
    300 sequences cross the offsets scan's 256-wide chunks."""
    rng = np.random.default_rng(800 + len(shape))
    B = 300
    lengths = rng.integers(0, 90, size=B)
    lengths[:5] = [0, 1, 89, 2, 0]
    nt = np.minimum(rng.integers(0, 6, size=B), lengths).astype(np.int32)
    off = _offsets(lengths)
    T = int(off[-1])
    if dtype == torch.int64:
        rows = torch.from_numpy(rng.integers(-2**62, 2**62, size=(T,) + shape))
    else:
        rows = torch.from_numpy(rng.standard_normal((T,) + shape).astype(np.float32)).to(dtype)
    for keep in (0, 1, 37, 200):
        _check_exact(off, nt, keep, rows, cuda_device)
    _check_exact(off, None, 13, rows, cuda_device)


def test_truncate_empty_inputs(cuda_device):
    # no sequences at all
    _check_exact(np.zeros(1, np.int64), None, 4, torch.zeros((0, 4), dtype=torch.float32), cuda_device)
    # sequences that are all empty
    _check_exact(np.zeros(4, np.int64), np.zeros(3, np.int32), 4, torch.zeros((0, 4), dtype=torch.float32),
                 cuda_device)


def test_truncate_rejects_bad_arguments(cuda_device):
    off = torch.tensor([0, 3], dtype=torch.int64, device=cuda_device)
    with pytest.raises(ops.HstuError):  # 2-byte rows
        ops.hstu_jagged_truncate(off, None, 1, torch.zeros(3, dtype=torch.bfloat16, device=cuda_device))
    with pytest.raises(ops.HstuError):  # negative segment length
        ops.hstu_jagged_truncate(off, None, -1, torch.zeros((3, 4), dtype=torch.float32, device=cuda_device))
    big = torch.zeros(3 * 8 + 1, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ops.HstuError):  # 16-byte rows at an address that is not 16-byte aligned
        ops.hstu_jagged_truncate(off, None, 1, big[1:].view(3, 8))


def _layer_kw(w, max_seq_len, attn):
    return dict(num_heads=w.num_heads, d_qk=w.d_qk, d_v=w.d_v, max_seq_len=max_seq_len, inv_n=attn.inv_n,
                pos_lo=attn.pos_lo, pos_hi=attn.pos_hi)


def _gpu_layer(x, lw, off, ts, nt, attn, w, max_seq_len, dev):
    return ops.hstu_layer_fwd(x, to_dev(lw.w1, dev), to_dev(lw.b1, dev), to_dev(lw.w2, dev), to_dev(lw.b2, dev),
                              to_dev(lw.ln_gamma, dev), to_dev(lw.ln_beta, dev), off, ts, nt,
                              to_dev(attn.rab_pos, dev), to_dev(attn.rab_time, dev), **_layer_kw(w, max_seq_len, attn))


def _oracle_layer(x, lw, off, ts, nt, attn, w):
    return oracle.layer_fwd(off, ts, nt, x, lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta, attn.rab_pos,
                            attn.rab_time, attn.pos_lo, attn.pos_hi, attn.inv_n, w.num_heads, w.d_qk, w.d_v)


def test_truncated_stack_small(cuda_device):
    """Two layers over whole histories, the cut, two layers over the kept
    segments (ragged, with candidates).  Each layer's oracle is fed the GPU's
    own input to that layer; the cut itself is compared bit for bit."""
    dev = cuda_device
    rng = np.random.default_rng(820)
    lengths = [150, 1, 70, 0, 260, 33]
    nt = [10, 0, 0, 0, 7, 33]
    attn = workloads.make_attn_inputs(rng, lengths, 2, 64, 64, 300.0, -200, 200, 32, 256, torch.bfloat16,
                                      num_targets=nt, with_values=False)
    w = workloads.Workload("t", 99, "bf16", len(lengths), "uniform", 1, 260, 2, 64, 64, 300.0, -200, 200, 32,
                           256, d_model=128)
    layers = [workloads.make_layer_weights(rng, 128, 2, 64, 64, torch.bfloat16, weight_std=0.1,
                                           random_affine=True) for _ in range(4)]
    x = torch.from_numpy(rng.standard_normal((attn.total_tokens, 128)).astype(np.float32)).to(torch.bfloat16)
    off, ts, ntd = (to_dev(t, dev) for t in (attn.seq_offsets, attn.timestamps, attn.num_targets))
    xg = to_dev(x, dev)
    for li in range(2):
        ref = _oracle_layer(xg.cpu(), layers[li], attn.seq_offsets, attn.timestamps, attn.num_targets, attn, w)
        xg = _gpu_layer(xg, layers[li], off, ts, ntd, attn, w, attn.max_seq_len, dev)
        assert_bf16_close(xg, ref, what=f"full layer {li}")
    keep = 48
    new_off, xk = ops.hstu_jagged_truncate(off, ntd, keep, xg)
    _, tk = ops.hstu_jagged_truncate(off, ntd, keep, ts)
    torch.cuda.synchronize()
    ref_off, ref_x = oracle.jagged_truncate(attn.seq_offsets, attn.num_targets, keep, xg.cpu().view(torch.int16).numpy())
    _, ref_t = oracle.jagged_truncate(attn.seq_offsets, attn.num_targets, keep, attn.timestamps.numpy())
    h_off = new_off.cpu().numpy()
    np.testing.assert_array_equal(h_off, ref_off)
    Tk = int(h_off[-1])
    np.testing.assert_array_equal(xk[:Tk].cpu().view(torch.int16).numpy(), ref_x)
    np.testing.assert_array_equal(tk[:Tk].cpu().numpy(), ref_t)
    xk, tk = xk[:Tk].contiguous(), tk[:Tk].contiguous()
    max_len = int(np.diff(h_off).max())
    for li in range(2, 4):
        ref = _oracle_layer(xk.cpu(), layers[li], h_off, tk.cpu().numpy(), attn.num_targets, attn, w)
        xk = _gpu_layer(xk, layers[li], new_off, tk, ntd, attn, w, max_len, dev)
        assert_bf16_close(xk, ref, what=f"segment layer {li}")


def test_truncate_layer_stack_batch(cuda_device):
    """The eight-layer stack's batch (64 Zipf-length histories up to 4096,
    D = 512) cut to its last 512 tokens: offsets and all kept rows bit-exact;
    one layer on the kept batch checked on three sequences by the oracle."""
    dev = cuda_device
    w = workloads.WORKLOADS["layer_stack_bf16"]
    inp = workloads.generate(w)
    attn = inp.attn
    keep = 512
    off, ts = to_dev(attn.seq_offsets, dev), to_dev(attn.timestamps, dev)
    new_off, xk = ops.hstu_jagged_truncate(off, None, keep, to_dev(inp.x, dev))
    _, tk = ops.hstu_jagged_truncate(off, None, keep, ts)
    torch.cuda.synchronize()
    ref_off, ref_x = oracle.jagged_truncate(attn.seq_offsets, None, keep, inp.x.view(torch.int16).numpy())
    h_off = new_off.cpu().numpy()
    np.testing.assert_array_equal(h_off, ref_off)
    Tk = int(h_off[-1])
    np.testing.assert_array_equal(xk[:Tk].cpu().view(torch.int16).numpy(), ref_x)
    xk, tk = xk[:Tk].contiguous(), tk[:Tk].contiguous()
    lens = np.diff(h_off)
    y = _gpu_layer(xk, inp.layers[0], new_off, tk, None, attn, w, int(lens.max()), dev)
    torch.cuda.synchronize()
    seqs = [int(np.argmax(lens)), int(np.argmin(lens)), len(lens) // 2]

    class _Kept:
        seq_offsets = torch.from_numpy(h_off)

    rows = rows_of(_Kept, seqs)
    sub_off = _offsets(lens[seqs])
    rows_t = torch.from_numpy(rows)
    ref = _oracle_layer(xk.cpu()[rows_t], inp.layers[0], sub_off, tk.cpu()[rows_t].numpy(), None, attn, w)
    assert_bf16_close(y[rows_t.to(dev)], ref, what="layer on the kept batch")
