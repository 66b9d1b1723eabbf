"""GPU parity of the transduction-layer backward against the CPU oracle (C ABI).

The GPU backward takes the GPU forward's saved tensors (bf16); the oracle
recomputes everything in fp64 from the same inputs.  Every output is compared
per tensor at the bf16 tolerance (max |gpu - oracle| <= 2e-2 max |oracle|)."""

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, to_dev

pytestmark = pytest.mark.gpu

NAMES = ["dx", "dw1", "db1", "dw2", "db2", "d_ln_gamma", "d_ln_beta", "d_rab_pos", "d_rab_time"]


def _case(seed, lengths, num_targets, H, d, D, pos, nb, weight_std):
    rng = np.random.default_rng(seed)
    attn = workloads.make_attn_inputs(rng, lengths, H, d, d, 300.0, -pos, pos, nb, max(lengths),
                                      torch.bfloat16, num_targets=num_targets, with_values=False)
    lw = workloads.make_layer_weights(rng, D, H, d, d, torch.bfloat16, weight_std=weight_std,
                                      random_affine=True)
    T = attn.total_tokens
    x = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(torch.bfloat16)
    dy = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(torch.bfloat16)
    return attn, lw, x, dy


def _run(attn, lw, x, dy, H, d, dev):
    kw = dict(num_heads=H, d_qk=d, d_v=d, max_seq_len=attn.max_seq_len, inv_n=attn.inv_n,
              pos_lo=attn.pos_lo, pos_hi=attn.pos_hi)
    T = x.shape[0]
    W = H * 4 * d
    xd = to_dev(x, dev)
    prm = [to_dev(t, dev) for t in (lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta)]
    seq = [to_dev(t, dev) for t in (attn.seq_offsets, attn.timestamps, attn.num_targets, attn.rab_pos,
                                   attn.rab_time)]
    uvqk = torch.empty((T, W), dtype=torch.bfloat16, device=dev)
    o = torch.empty((T, H * d), dtype=torch.bfloat16, device=dev)
    ops.hstu_layer_fwd(xd, *prm, *seq, saved_uvqk=uvqk, saved_o=o, **kw)
    w1, b1, w2, _, g, be = prm
    grads = ops.hstu_layer_bwd(xd, w1, b1, w2, g, be, *seq, uvqk, o, to_dev(dy, dev), **kw)
    torch.cuda.synchronize()
    ref = oracle.layer_bwd(attn.seq_offsets, attn.timestamps, attn.num_targets, x, lw.w1, lw.b1, lw.w2,
                           lw.ln_gamma, lw.ln_beta, attn.rab_pos, attn.rab_time, attn.pos_lo, attn.pos_hi,
                           attn.inv_n, H, d, d, dy)
    return grads, ref


def _check(grads, ref):
    for n in NAMES:
        assert_bf16_close(grads[n], ref[n], what=n)


def test_layer_bwd_small_ragged_candidates(cuda_device):
    # D = 128, 2 heads of 64: H d_v = 128, W = 512; 236 tokens (the weight-gradient
    # GEMMs' token dimension is not a multiple of 64), an empty and a one-token sequence
    attn, lw, x, dy = _case(71, [100, 1, 37, 0, 98], [10, 0, 0, 0, 3], 2, 64, 128, 200, 32, 0.1)
    grads, ref = _run(attn, lw, x, dy, 2, 64, cuda_device)
    _check(grads, ref)


def test_layer_bwd_stack_dims(cuda_device):
    # the layer-stack dimensions (D = 512, 4 heads of 128, W = 2048) on a Zipf-like
    # mix of short and long sequences, 3,1xx tokens
    attn, lw, x, dy = _case(72, [1500, 32, 900, 32, 611, 97], None, 4, 128, 512, 4096, 128, 0.05)
    grads, ref = _run(attn, lw, x, dy, 4, 128, cuda_device)
    _check(grads, ref)


def test_layer_bwd_rejects_unsupported(cuda_device):
    # D not a multiple of 128: reported, nothing launched
    attn, lw, x, dy = _case(73, [20, 5], None, 2, 64, 96, 50, 16, 0.1)
    with pytest.raises(RuntimeError):
        _run(attn, lw, x, dy, 2, 64, cuda_device)
