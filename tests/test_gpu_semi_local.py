"""GPU parity of semi-local attention (local + global windows) against the CPU oracle.

Every kernel path sees the windows: tcgen05 (d = 64, 128, forward and
backward) and fp32."""

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import workloads
from parity_utils import assert_bf16_close, assert_f32_close, gpu_bwd, gpu_fwd

pytestmark = pytest.mark.gpu

NAMES = ["dq", "dk", "dv", "d_rab_pos", "d_rab_time"]


def _inp(lengths, nt, d, seed, dtype=torch.bfloat16, lo=-300, hi=300, n_scale=512, gap=300.0):
    rng = np.random.default_rng(seed)
    return workloads.make_attn_inputs(rng, lengths, 2, d, d, gap, lo, hi, 32, n_scale, dtype,
                                      num_targets=nt, with_dout=True)


def _args(inp):
    return (inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v, inp.rab_pos,
            inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n)


# windows: a band narrower than a tile, one crossing tiles with a global prefix that is
# not tile aligned, and one wider than most sequences
WINDOWS = [(70, 0), (200, 130), (1000, 64)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lw,gw", WINDOWS)
def test_semi_local_fwd_bwd_ragged(cuda_device, d, lw, gw):
    inp = _inp([1, 0, 300, 77, 513, 129], [0, 0, 10, 0, 40, 1], d, seed=600 + d + lw)
    win = dict(local_window=lw, global_window=gw)
    assert_bf16_close(gpu_fwd(inp, cuda_device, **win), oracle.attn_fwd(*_args(inp), **win),
                      what=f"fwd d={d} w=({lw},{gw})")
    g = gpu_bwd(inp, cuda_device, **win)
    r = oracle.attn_bwd(*_args(inp), inp.dout, **win)
    for n, a, b in zip(NAMES, g, r):
        assert_bf16_close(a, b, what=f"bwd d={d} w=({lw},{gw}) {n}")


def test_semi_local_f32(cuda_device):
    inp = _inp([1, 70, 128, 33], [0, 3, 0, 2], 32, seed=650, dtype=torch.float32, lo=0, hi=127, n_scale=128,
               gap=60.0)
    win = dict(local_window=20, global_window=5)
    assert_f32_close(gpu_fwd(inp, cuda_device, **win), oracle.attn_fwd(*_args(inp), **win), what="fwd f32")
    g = gpu_bwd(inp, cuda_device, **win)
    r = oracle.attn_bwd(*_args(inp), inp.dout, **win)
    for n, a, b in zip(NAMES, g, r):
        assert_f32_close(a, b, what=f"bwd f32 {n}")


def test_semi_local_wide_window_is_full(cuda_device):
    # a local window covering every distance reproduces the full mask bit for bit
    inp = _inp([300, 129], [10, 0], 128, seed=660)
    full = gpu_fwd(inp, cuda_device)
    wide = gpu_fwd(inp, cuda_device, local_window=1 << 20, global_window=0)
    assert torch.equal(full, wide)


def test_semi_local_long_history_sampled(cuda_device):
    # long-history shapes (two sequences of 8-16k), local 1024, global 256
    w = workloads.WORKLOADS["long_history_bf16"]
    rng = np.random.default_rng(w.seed + 5)
    inp = workloads.make_attn_inputs(rng, [16000, 9000], 4, 128, 128, 300.0, -4096, 4096, 128, 16384,
                                     torch.bfloat16, with_dout=True)
    win = dict(local_window=1024, global_window=256)
    out = gpu_fwd(inp, cuda_device, **win)
    dq, dk, dv, drp, drt = gpu_bwd(inp, cuda_device, **win)
    rows = np.array([0, 255, 256, 1023, 1024, 1100, 5000, 15999, 16000, 16255, 17100, 24999], dtype=np.int64)
    ref = oracle.attn_fwd_rows(*_args(inp), rows, **win)
    dev = cuda_device
    assert_bf16_close(out[torch.from_numpy(rows).to(dev)], ref, what="semi-local long fwd rows")
    rq, rk, rv = oracle.attn_bwd_rows(*_args(inp), inp.dout, rows, rows, **win)
    idx = torch.from_numpy(rows).to(dev)
    assert_bf16_close(dq[idx], rq, what="semi-local long dq rows")
    assert_bf16_close(dk[idx], rk, what="semi-local long dk rows")
    assert_bf16_close(dv[idx], rv, what="semi-local long dv rows")
    tp, tt = float(drp.double().sum()), float(drt.double().sum())
    assert abs(tp - tt) <= 1e-3 * max(abs(tp), float(drp.abs().sum())), (tp, tt)


def test_semi_local_layer_fwd_bwd(cuda_device):
    """One bf16 layer (D = 128, 2 heads of 64) forward and backward with the
    windows, against the oracle's windowed layer."""
    import oracle as _oracle
    from hstu_sequential_transduction_b200 import ops as _ops
    from parity_utils import assert_bf16_close, to_dev
    rng = np.random.default_rng(760)
    attn = workloads.make_attn_inputs(rng, [300, 1, 90, 0, 257], 2, 64, 64, 300.0, -400, 400, 32, 300,
                                      torch.bfloat16, num_targets=[20, 0, 0, 0, 7], with_values=False)
    lw = workloads.make_layer_weights(rng, 128, 2, 64, 64, torch.bfloat16, weight_std=0.1, random_affine=True)
    T = attn.total_tokens
    x = torch.from_numpy(rng.standard_normal((T, 128)).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy(rng.standard_normal((T, 128)).astype(np.float32)).to(torch.bfloat16)
    dev = cuda_device
    win = dict(local_window=64, global_window=16)
    kw = dict(num_heads=2, d_qk=64, d_v=64, max_seq_len=attn.max_seq_len, inv_n=attn.inv_n, pos_lo=attn.pos_lo,
              pos_hi=attn.pos_hi, **win)
    prm = [to_dev(t, dev) for t in (lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta)]
    seq = [to_dev(t, dev) for t in (attn.seq_offsets, attn.timestamps, attn.num_targets, attn.rab_pos, attn.rab_time)]
    uvqk = torch.empty((T, 512), dtype=torch.bfloat16, device=dev)
    o = torch.empty((T, 128), dtype=torch.bfloat16, device=dev)
    y = _ops.hstu_layer_fwd(to_dev(x, dev), *prm, *seq, saved_uvqk=uvqk, saved_o=o, **kw)
    w1, b1, w2, _, g, be = prm
    grads = _ops.hstu_layer_bwd(to_dev(x, dev), w1, b1, w2, g, be, *seq, uvqk, o, to_dev(dy, dev), **kw)
    torch.cuda.synchronize()
    oargs = (attn.seq_offsets, attn.timestamps, attn.num_targets)
    ref = _oracle.layer_fwd(*oargs, x, lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta, attn.rab_pos,
                            attn.rab_time, attn.pos_lo, attn.pos_hi, attn.inv_n, 2, 64, 64, **win)
    assert_bf16_close(y, ref, what="windowed layer output")
    refg = _oracle.layer_bwd(*oargs, x, lw.w1, lw.b1, lw.w2, lw.ln_gamma, lw.ln_beta, attn.rab_pos, attn.rab_time,
                             attn.pos_lo, attn.pos_hi, attn.inv_n, 2, 64, 64, dy, **win)
    for n in ("dx", "dw1", "db1", "dw2", "db2", "d_ln_gamma", "d_ln_beta", "d_rab_pos", "d_rab_time"):
        assert_bf16_close(grads[n], refg[n], what=n)
