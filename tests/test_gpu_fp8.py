"""GPU parity of the FP8 (E4M3) projections against the oracle: the quantisers
bit for bit (codes and float32 scales, the sign of a zero code aside), the
tcgen05 kind::f8f6f4 GEMM against the oracle's float64 product of its own
codes, and the layer with FP8 projections against the oracle's FP8 layer."""

import ctypes

import numpy as np
import pytest
import torch

from oracle import fp8 as ofp8
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, rows_of, to_dev

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, scale=1.0):
    return torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16)


def _same_codes(got, ref):
    got, ref = np.asarray(got, np.uint8), np.asarray(ref, np.uint8)
    zero = (ref & 0x7F) == 0
    np.testing.assert_array_equal(got & 0x7F, ref & 0x7F)          # magnitudes everywhere
    np.testing.assert_array_equal(got[~zero], ref[~zero])          # signs of non-zero codes


def test_quantize_rows_bit_exact(cuda_device):
    rng = np.random.default_rng(1000)
    R, K = 300, 512
    x = _bf16(rng, (R, K)) * torch.from_numpy(np.exp2(rng.integers(-12, 12, (R, 1))).astype(np.float32)).to(
        torch.bfloat16)
    x[5] = 0
    x[6, 17] = 3.0e4  # one large value: the rest of the row lands in subnormal codes
    codes, scales = ops.quantize_rows_e4m3(x.to(cuda_device))
    torch.cuda.synchronize()
    ref_c, ref_s = ofp8.quantize_rows(x.float().numpy())
    _same_codes(codes.cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)


def test_quantize_weight_bit_exact(cuda_device):
    rng = np.random.default_rng(1001)
    K, N = 512, 384
    w = _bf16(rng, (K, N), 0.02)
    w[:, 7] = 0
    pack = ops.quantize_weight_e4m3(w.to(cuda_device))
    torch.cuda.synchronize()
    codes, scales = ops.e4m3_pack_parts(pack, K, N)
    ref_c, ref_s = ofp8.quantize_weight(w.float().numpy())
    _same_codes(codes.cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)


@pytest.mark.parametrize("M,K,N,silu", [(1000, 512, 384, True), (257, 128, 512, False), (64, 2048, 256, True)])
def test_gemm_e4m3_matches_oracle(cuda_device, M, K, N, silu):
    rng = np.random.default_rng(1002 + M)
    x = _bf16(rng, (M, K))
    w = _bf16(rng, (K, N), 0.05)
    b = _bf16(rng, (N,), 0.1)
    codes, scales = ops.quantize_rows_e4m3(x.to(cuda_device))
    pack = ops.quantize_weight_e4m3(w.to(cuda_device))
    y = ops.gemm_e4m3(codes, scales, pack, N, bias=b.to(cuda_device), apply_silu=silu)
    torch.cuda.synchronize()
    xq, sx = ofp8.quantize_rows(x.float().numpy())
    wq, sw = ofp8.quantize_weight(w.float().numpy())
    ref = ofp8.gemm(xq, sx, wq, sw, b.float().numpy(), apply_silu=silu)
    # same codes on both sides: only float32 accumulation and the bf16 output differ
    assert_bf16_close(y, ref, tol=8e-3, what="E4M3 GEMM")


# The layer's G is quantised from values that differ between the two sides by
# bf16 rounding upstream (~2^-8 relative), so a few percent of its E4M3 codes
# (spacing 2^-3 to 2^-4 relative) land one code apart; summed over the H d_v
# inputs of f2 those flips give ~0.5 % of the output's max-abs typically and
# ~2.5 % at the extreme element.  The layer test allows twice that; the
# quantisers (bit-exact) and the GEMM (8e-3) are checked on their own above.
FP8_LAYER_TOL = 5e-2


def _layer_case(seed, lengths, nt, H, d, D, pos, nb):
    rng = np.random.default_rng(seed)
    attn = workloads.make_attn_inputs(rng, lengths, H, d, d, 300.0, -pos, pos, nb, max(lengths), torch.bfloat16,
                                      num_targets=nt, with_values=False)
    lw = workloads.make_layer_weights(rng, D, H, d, d, torch.bfloat16, weight_std=0.1, random_affine=True)
    x = _bf16(rng, (attn.total_tokens, D))
    return attn, lw, x


def _bf16_round(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).double().numpy()


def _run_fp8_layer(attn, lw, x, H, d, dev, rows=None):
    T = x.shape[0]
    W = H * 4 * d
    p1 = ops.quantize_weight_e4m3(to_dev(lw.w1, dev))
    p2 = ops.quantize_weight_e4m3(to_dev(lw.w2, dev))
    seq = [to_dev(t, dev) for t in (attn.seq_offsets, attn.timestamps, attn.num_targets, attn.rab_pos,
                                   attn.rab_time)]
    uvqk = torch.empty((T, W), dtype=torch.bfloat16, device=dev)
    y = ops.hstu_layer_fwd(to_dev(x, dev), p1, to_dev(lw.b1, dev), p2, to_dev(lw.b2, dev), to_dev(lw.ln_gamma, dev),
                           to_dev(lw.ln_beta, dev), *seq, num_heads=H, d_qk=d, d_v=d, max_seq_len=attn.max_seq_len,
                           inv_n=attn.inv_n, pos_lo=attn.pos_lo, pos_hi=attn.pos_hi, fp8_projections=True,
                           saved_uvqk=uvqk)
    torch.cuda.synchronize()
    w1q, s1 = ofp8.quantize_weight(lw.w1.float().numpy())
    w2q, s2 = ofp8.quantize_weight(lw.w2.float().numpy())
    off, ts, nt = attn.seq_offsets, attn.timestamps, attn.num_targets
    xs = x
    if rows is not None:  # a sub-batch of whole sequences (sequences are independent)
        seqs, sub_off = rows
        idx = torch.from_numpy(rows_of(attn, seqs))
        off, ts, xs = sub_off, attn.timestamps[idx], x[idx]
        nt = None if nt is None else nt[list(seqs)]
        y, uvqk = y[idx.to(dev)], uvqk[idx.to(dev)]
    ref, ref_uvqk, _ = ofp8.layer_fwd(off, ts, nt, xs.float().numpy(), w1q, s1, lw.b1.float().numpy(), w2q, s2,
                                      lw.b2.float().numpy(), lw.ln_gamma, lw.ln_beta, attn.rab_pos, attn.rab_time,
                                      attn.pos_lo, attn.pos_hi, attn.inv_n, H, d, d, g_round=_bf16_round,
                                      want_intermediates=True)
    # X is quantised identically on both sides: f1's output is held to the GEMM's tolerance
    assert_bf16_close(uvqk, ref_uvqk, tol=8e-3, what="FP8 f1 output (U|V|Q|K)")
    return y, ref


def test_fp8_layer_small_ragged(cuda_device):
    # D = 128, 2 heads of 64, candidates, an empty and a one-token sequence
    attn, lw, x = _layer_case(1010, [100, 1, 37, 0, 130], [10, 0, 0, 0, 3], 2, 64, 128, 200, 32)
    y, ref = _run_fp8_layer(attn, lw, x, 2, 64, cuda_device)
    assert_bf16_close(y, ref, tol=FP8_LAYER_TOL, what="FP8 layer output")


def test_fp8_layer_stack_dims(cuda_device):
    # the layer-stack dimensions (D = 512, 4 heads of 128) on a Zipf-like mix; the
    # oracle recomputes three of the sequences
    lengths = [1500, 32, 900, 32, 611, 97]
    attn, lw, x = _layer_case(1011, lengths, None, 4, 128, 512, 4096, 128)
    seqs = [1, 4, 5]
    sub_off = np.concatenate([[0], np.cumsum(np.asarray(lengths)[seqs])]).astype(np.int64)
    y, ref = _run_fp8_layer(attn, lw, x, 4, 128, cuda_device, rows=(seqs, sub_off))
    assert_bf16_close(y, ref, tol=FP8_LAYER_TOL, what="FP8 layer output")


def test_fp8_rejects_unsupported(cuda_device):
    x = torch.zeros((8, 24), dtype=torch.bfloat16, device=cuda_device)  # K not a multiple of 16
    with pytest.raises(ops.HstuError):
        ops.quantize_rows_e4m3(x)
    codes = torch.zeros((8, 32), dtype=torch.uint8, device=cuda_device)
    scales = torch.ones(8, dtype=torch.float32, device=cuda_device)
    pack = torch.zeros(ops.hstu_e4m3_weight_bytes(32, 100), dtype=torch.uint8, device=cuda_device)
    with pytest.raises(ops.HstuError):  # N not a multiple of 128
        ops.gemm_e4m3(codes, scales, pack, 100)


def _fp8_attn_case(seed, lengths, nt, H=2, pos=300, nb=32):
    rng = np.random.default_rng(seed)
    return workloads.make_attn_inputs(rng, lengths, H, 128, 128, 300.0, -pos, pos, nb, max(lengths), torch.bfloat16,
                                      num_targets=nt)


@pytest.mark.parametrize("windows", [{}, {"local_window": 100, "global_window": 20}])
def test_fp8_score_attention_matches_oracle(cuda_device, windows):
    """Q K^T on E4M3 codes (q, k quantised per (token, head) row inside the
    call): ragged batch with candidates, an empty and a one-token sequence."""
    inp = _fp8_attn_case(1020, [300, 1, 0, 257, 129], [20, 0, 0, 0, 9])
    dev = cuda_device
    d = {k: (None if getattr(inp, k) is None else getattr(inp, k).to(dev))
         for k in ("q", "k", "v", "seq_offsets", "timestamps", "num_targets", "rab_pos", "rab_time")}
    out = ops.hstu_attn_fwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["num_targets"],
                            d["rab_pos"], d["rab_time"], max_seq_len=inp.max_seq_len, inv_n=inp.inv_n,
                            pos_lo=inp.pos_lo, pos_hi=inp.pos_hi, fp8_qk=True, **windows)
    torch.cuda.synchronize()
    ref = ofp8.attn_fwd_qk(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v, inp.rab_pos,
                           inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, **windows)
    assert_bf16_close(out, ref, what="FP8-score attention")


def test_fp8_score_attention_rejections(cuda_device):
    inp = _fp8_attn_case(1021, [64, 30], None)
    dev = cuda_device
    d = {k: (None if getattr(inp, k) is None else getattr(inp, k).to(dev))
         for k in ("q", "k", "v", "seq_offsets", "timestamps", "rab_pos", "rab_time")}
    kw = dict(max_seq_len=inp.max_seq_len, inv_n=inp.inv_n, pos_lo=inp.pos_lo, pos_hi=inp.pos_hi)
    # d = 64: not supported with FP8 scores
    q64 = d["q"][..., :64].contiguous()
    with pytest.raises(ops.HstuError):
        ops.hstu_attn_fwd(q64, q64, q64, d["seq_offsets"], d["timestamps"], None, d["rab_pos"], d["rab_time"],
                          fp8_qk=True, **kw)
    # the backward rejects the option
    desc = ops._attn_desc_from(d["q"], d["v"], d["seq_offsets"], inp.max_seq_len, inp.inv_n, inp.pos_lo,
                               inp.pos_hi, d["rab_pos"], d["rab_time"], fp8_qk=True)
    n = ctypes.c_size_t(0)
    assert ops.load_library().hstu_attn_workspace_size(ctypes.byref(desc), 1, ctypes.byref(n)) == 0
    ws = ops.alloc_workspace(n.value, dev)
    g = [torch.empty_like(d["q"]) for _ in range(3)] + [torch.empty_like(d["rab_pos"]), torch.empty_like(d["rab_time"])]
    st = ops.load_library().hstu_attn_bwd(
        ctypes.byref(desc), ops._ptr(d["q"]), ops._ptr(d["k"]), ops._ptr(d["v"]), ops._ptr(d["seq_offsets"]),
        ops._ptr(d["timestamps"]), None, ops._ptr(d["rab_pos"]), ops._ptr(d["rab_time"]), ops._ptr(d["q"]),
        *[ops._ptr(t) for t in g], ops._ptr(ws), ctypes.c_size_t(ws.numel()), None)
    assert st == 2  # HSTU_ERR_UNSUPPORTED
