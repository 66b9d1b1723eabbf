"""GPU parity of the layer whose output projection reads [U | O | G] (3 H d_v
wide) against the oracle's same variant: forward on the tcgen05 path (the
GEMM reads the three blocks from their own buffers), on the copy paths (fp32,
and bf16 with D not a multiple of 128), and the layer backward."""

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, assert_f32_close, to_dev

pytestmark = pytest.mark.gpu

NAMES = ["dx", "dw1", "db1", "dw2", "db2", "d_ln_gamma", "d_ln_beta", "d_rab_pos", "d_rab_time"]


def _w2_cat(rng, H, d, D, std, dtype):
    return torch.from_numpy(rng.standard_normal((3 * H * d, D)).astype(np.float32) * std).to(dtype)


def _case(seed, lengths, num_targets, H, d, D, pos, nb, weight_std, dtype=torch.bfloat16):
    rng = np.random.default_rng(seed)
    attn = workloads.make_attn_inputs(rng, lengths, H, d, d, 300.0, -pos, pos, nb, max(lengths), dtype,
                                      num_targets=num_targets, with_values=False)
    lw = workloads.make_layer_weights(rng, D, H, d, d, dtype, weight_std=weight_std, random_affine=True)
    w2 = _w2_cat(rng, H, d, D, weight_std, dtype)
    T = attn.total_tokens
    x = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(dtype)
    dy = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32)).to(dtype)
    return attn, lw, w2, x, dy


def _kw(attn, H, d):
    return dict(num_heads=H, d_qk=d, d_v=d, max_seq_len=attn.max_seq_len, inv_n=attn.inv_n, pos_lo=attn.pos_lo,
                pos_hi=attn.pos_hi, output_concat=True)


def _fwd(attn, lw, w2, x, H, d, dev, saved=False):
    T = x.shape[0]
    seq = [to_dev(t, dev) for t in (attn.seq_offsets, attn.timestamps, attn.num_targets, attn.rab_pos,
                                   attn.rab_time)]
    uvqk = torch.empty((T, H * 4 * d), dtype=x.dtype, device=dev) if saved else None
    o = torch.empty((T, H * d), dtype=x.dtype, device=dev) if saved else None
    y = ops.hstu_layer_fwd(to_dev(x, dev), to_dev(lw.w1, dev), to_dev(lw.b1, dev), to_dev(w2, dev),
                           to_dev(lw.b2, dev), to_dev(lw.ln_gamma, dev), to_dev(lw.ln_beta, dev), *seq,
                           saved_uvqk=uvqk, saved_o=o, **_kw(attn, H, d))
    torch.cuda.synchronize()
    return y, uvqk, o, seq


def _oracle_fwd(attn, lw, w2, x, H, d):
    return oracle.layer_fwd(attn.seq_offsets, attn.timestamps, attn.num_targets, x, lw.w1, lw.b1, w2, lw.b2,
                            lw.ln_gamma, lw.ln_beta, attn.rab_pos, attn.rab_time, attn.pos_lo, attn.pos_hi,
                            attn.inv_n, H, d, d, out_cat=True)


def test_concat_fwd_f32_small(cuda_device):
    # fp32, D = 64, 2 heads of 32: the concatenation is copied, then the fp32 GEMM
    attn, lw, w2, x, _ = _case(90, [16, 100, 57, 128], None, 2, 32, 64, 64, 32, 0.1, torch.float32)
    y, _, _, _ = _fwd(attn, lw, w2, x, 2, 32, cuda_device)
    assert_f32_close(y, _oracle_fwd(attn, lw, w2, x, 2, 32), what="layer output")


def test_concat_fwd_bf16_tcgen05(cuda_device):
    # D = 128, H d_v = 128: the tcgen05 GEMM reads U, O and G from their buffers
    attn, lw, w2, x, _ = _case(91, [100, 1, 37, 0, 130], [10, 0, 0, 0, 3], 2, 64, 128, 200, 32, 0.1)
    y, _, _, _ = _fwd(attn, lw, w2, x, 2, 64, cuda_device)
    assert_bf16_close(y, _oracle_fwd(attn, lw, w2, x, 2, 64), what="layer output")


def test_concat_fwd_bf16_partial_column_tile(cuda_device):
    # D = 96 is not a multiple of the GEMM's 128-column tile: the tcgen05 GEMM reads
    # [U | O | G] from the three buffers and its one column tile is partial
    attn, lw, w2, x, _ = _case(92, [70, 3, 129], [5, 0, 9], 2, 64, 96, 100, 16, 0.1)
    y, _, _, _ = _fwd(attn, lw, w2, x, 2, 64, cuda_device)
    assert_bf16_close(y, _oracle_fwd(attn, lw, w2, x, 2, 64), what="layer output")


def _bwd(seed, lengths, num_targets, H, d, D, pos, nb, weight_std, dev):
    attn, lw, w2, x, dy = _case(seed, lengths, num_targets, H, d, D, pos, nb, weight_std)
    y, uvqk, o, seq = _fwd(attn, lw, w2, x, H, d, dev, saved=True)
    assert_bf16_close(y, _oracle_fwd(attn, lw, w2, x, H, d), what="layer output")
    grads = ops.hstu_layer_bwd(to_dev(x, dev), to_dev(lw.w1, dev), to_dev(lw.b1, dev), to_dev(w2, dev),
                               to_dev(lw.ln_gamma, dev), to_dev(lw.ln_beta, dev), *seq, uvqk, o, to_dev(dy, dev),
                               **_kw(attn, H, d))
    torch.cuda.synchronize()
    ref = oracle.layer_bwd(attn.seq_offsets, attn.timestamps, attn.num_targets, x, lw.w1, lw.b1, w2, lw.ln_gamma,
                           lw.ln_beta, attn.rab_pos, attn.rab_time, attn.pos_lo, attn.pos_hi, attn.inv_n, H, d, d,
                           dy, out_cat=True)
    for n in NAMES:
        assert_bf16_close(grads[n], ref[n], what=n)


def test_concat_bwd_small_ragged_candidates(cuda_device):
    # 236 tokens, an empty and a one-token sequence; dW2 is [384, 128]
    _bwd(93, [100, 1, 37, 0, 98], [10, 0, 0, 0, 3], 2, 64, 128, 200, 32, 0.1, cuda_device)


def test_concat_bwd_stack_dims(cuda_device):
    # D = 512, 4 heads of 128: [U | O | G] is 1536 wide
    _bwd(94, [1500, 32, 900, 32, 611, 97], None, 4, 128, 512, 4096, 128, 0.05, cuda_device)


def test_concat_rejects_w2_of_the_wrong_height(cuda_device):
    attn, lw, w2, x, _ = _case(95, [20, 5], None, 2, 64, 128, 50, 16, 0.1)
    with pytest.raises(ValueError):
        ops.hstu_layer_fwd(to_dev(x, cuda_device), to_dev(lw.w1, cuda_device), to_dev(lw.b1, cuda_device),
                           to_dev(lw.w2, cuda_device), to_dev(lw.b2, cuda_device), to_dev(lw.ln_gamma, cuda_device),
                           to_dev(lw.ln_beta, cuda_device), to_dev(attn.seq_offsets, cuda_device),
                           to_dev(attn.timestamps, cuda_device), None, to_dev(attn.rab_pos, cuda_device),
                           to_dev(attn.rab_time, cuda_device), **_kw(attn, 2, 64))
