"""GPU parity of the full transduction layer against the CPU oracle (C ABI)."""

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, assert_f32_close, rows_of, to_dev

pytestmark = pytest.mark.gpu


def _gpu_layer(x, lw, attn, w, dev, saved=False):
    kw = dict(num_heads=w.num_heads, d_qk=w.d_qk, d_v=w.d_v, max_seq_len=attn.max_seq_len,
              inv_n=attn.inv_n, pos_lo=attn.pos_lo, pos_hi=attn.pos_hi)
    T = x.shape[0]
    uvqk = o = None
    if saved:
        uvqk = torch.empty((T, w.num_heads * (2 * w.d_v + 2 * w.d_qk)), dtype=x.dtype, device=dev)
        o = torch.empty((T, w.num_heads * w.d_v), dtype=x.dtype, device=dev)
    y = ops.hstu_layer_fwd(x, to_dev(lw.w1, dev), to_dev(lw.b1, dev), to_dev(lw.w2, dev),
                           to_dev(lw.b2, dev), to_dev(lw.ln_gamma, dev), to_dev(lw.ln_beta, dev),
                           to_dev(attn.seq_offsets, dev), to_dev(attn.timestamps, dev),
                           to_dev(attn.num_targets, dev), to_dev(attn.rab_pos, dev),
                           to_dev(attn.rab_time, dev), saved_uvqk=uvqk, saved_o=o, **kw)
    torch.cuda.synchronize()
    return (y, uvqk, o) if saved else y


def _oracle_layer(x, lw, attn, w, off=None, ts=None, nt=None, inter=False):
    off = attn.seq_offsets if off is None else off
    ts = attn.timestamps if ts is None else ts
    nt = attn.num_targets if nt is None else nt
    return oracle.layer_fwd(off, ts, nt, x, lw.w1, lw.b1, lw.w2, lw.b2, lw.ln_gamma, lw.ln_beta,
                            attn.rab_pos, attn.rab_time, attn.pos_lo, attn.pos_hi, attn.inv_n,
                            w.num_heads, w.d_qk, w.d_v, want_intermediates=inter)


def test_layer_f32_small_full(cuda_device):
    w = workloads.WORKLOADS["layer_f32_small"]
    inp = workloads.generate(w)
    lw = inp.layers[0]
    y, uvqk, o = _gpu_layer(to_dev(inp.x, cuda_device), lw, inp.attn, w, cuda_device, saved=True)
    ry, ruvqk, ro = _oracle_layer(inp.x, lw, inp.attn, w, inter=True)
    assert_f32_close(uvqk, ruvqk, what="uvqk")
    assert_f32_close(o, ro, what="attention output")
    assert_f32_close(y, ry, what="layer output")


def test_layer_bf16_random_affine_ragged(cuda_device):
    rng = np.random.default_rng(42)
    attn = workloads.make_attn_inputs(rng, [100, 1, 37, 0, 130], 2, 64, 64, 300.0, -200, 200, 32,
                                      256, torch.bfloat16, num_targets=[10, 0, 0, 0, 3],
                                      with_values=False)
    w = workloads.Workload("t", 99, "bf16", 5, "uniform", 1, 130, 2, 64, 64, 300.0, -200, 200, 32,
                           256, d_model=128)
    lw = workloads.make_layer_weights(rng, 128, 2, 64, 64, torch.bfloat16, weight_std=0.1,
                                      random_affine=True)
    x = (torch.from_numpy(rng.standard_normal((attn.total_tokens, 128)).astype(np.float32))
         .to(torch.bfloat16))
    y, uvqk, o = _gpu_layer(to_dev(x, cuda_device), lw, attn, w, cuda_device, saved=True)
    ry, ruvqk, ro = _oracle_layer(x, lw, attn, w, inter=True)
    assert_bf16_close(uvqk, ruvqk, what="uvqk")
    assert_bf16_close(o, ro, what="attention output")
    assert_bf16_close(y, ry, what="layer output")


def _pick(lengths, lo, hi, k):
    idx = [i for i, L in enumerate(lengths) if lo <= L <= hi]
    return idx[:k]


# Below this magnitude a layer's intermediates leave the fp32/bf16 normal range.
REPRESENTABLE = 1e-30


def test_layer_stack_bf16_per_layer(cuda_device):
    """Eight-layer stack at full batch on the GPU; the oracle runs the same stack on
    a sub-batch of sequences (sequences are independent) and every layer's rows
    of those sequences are compared.

    The stack has no residual connection and its weights are N(0, 0.02), so the
    activations shrink roughly quadratically with depth (LayerNorm's eps
    dominates the variance of the tiny attention output): the oracle's layer
    outputs fall from ~1e-6 to ~1e-15, ~1e-34, ~1e-72.  Layers whose reference
    output and attention output are representable are held to the bf16
    tolerance; deeper layers must have underflowed on the GPU as well."""
    w = workloads.WORKLOADS["layer_stack_bf16"]
    inp = workloads.generate(w)
    attn = inp.attn
    lengths = attn.lengths
    seqs = sorted(set(_pick(lengths, 32, 32, 1) + _pick(lengths, 33, 400, 1) + _pick(lengths, 401, 1100, 1)))
    assert seqs
    rows = rows_of(attn, seqs)
    sub_len = lengths[seqs]
    sub_off = np.concatenate([[0], np.cumsum(sub_len)]).astype(np.int64)
    sub_ts = attn.timestamps[torch.from_numpy(rows)]
    x_gpu = to_dev(inp.x, cuda_device)
    x_ref = inp.x[torch.from_numpy(rows)]
    rows_dev = torch.from_numpy(rows).to(cuda_device)
    compared = 0
    for layer, lw in enumerate(inp.layers):
        x_gpu = _gpu_layer(x_gpu, lw, attn, w, cuda_device)
        x_ref, _, o_ref = _oracle_layer(x_ref, lw, attn, w, off=sub_off, ts=sub_ts, nt=None,
                                        inter=True)
        if np.abs(x_ref).max() >= REPRESENTABLE and np.abs(o_ref).max() >= REPRESENTABLE:
            assert_bf16_close(x_gpu[rows_dev], x_ref, what=f"layer {layer}")
            compared += 1
        else:
            assert float(x_gpu[rows_dev].abs().max()) <= REPRESENTABLE, f"layer {layer}"
    assert compared >= 2


def test_layer_stack_bf16_every_layer_representable(cuda_device):
    """The eight-layer stack of the Zipf-length batch (64 histories up to 4096
    tokens, D = 512, 4 heads of 128) at full batch on the GPU, with weights
    N(0, 0.06) and inputs N(0, 1) so that no layer underflows (the layer
    outputs stay between ~1 and ~100 in magnitude).  Every layer is compared:
    the oracle runs each layer on the rows of three sequences (32, ~300 and
    4096 tokens, the longest length of the batch) taking as input the same bf16
    values the GPU layer consumed, and its attention output O and layer output
    Y are held to the bf16 tolerance."""
    w = workloads.WORKLOADS["layer_stack_bf16"]
    inp = workloads.generate(w)
    attn = inp.attn
    lengths = attn.lengths
    seqs = sorted(set(_pick(lengths, 32, 32, 1) + _pick(lengths, 250, 400, 1) + _pick(lengths, 4096, 4096, 1)))
    assert len(seqs) == 3 and lengths[seqs].max() == 4096
    rows = rows_of(attn, seqs)
    sub_off = np.concatenate([[0], np.cumsum(lengths[seqs])]).astype(np.int64)
    sub_ts = attn.timestamps[torch.from_numpy(rows)]
    rng = np.random.default_rng(2024)
    layers = [workloads.make_layer_weights(rng, w.d_model, w.num_heads, w.d_qk, w.d_v, torch.bfloat16,
                                           weight_std=0.06) for _ in range(w.num_layers)]
    x = (torch.from_numpy(rng.standard_normal((attn.total_tokens, w.d_model)).astype(np.float32))
         .to(torch.bfloat16).to(cuda_device))
    rows_dev = torch.from_numpy(rows).to(cuda_device)
    for layer, lw in enumerate(layers):
        x_in = x[rows_dev].cpu()
        y, _, o = _gpu_layer(x, lw, attn, w, cuda_device, saved=True)
        ry, _, ro = _oracle_layer(x_in, lw, attn, w, off=sub_off, ts=sub_ts, nt=None, inter=True)
        assert np.abs(ry).max() > 1e-1, f"layer {layer} degenerated"
        assert_bf16_close(o[rows_dev], ro, what=f"layer {layer} attention output")
        assert_bf16_close(y[rows_dev], ry, what=f"layer {layer} output")
        x = y


def test_ranking_layer_one_user(cuda_device):
    """Ranking layer (2048 history + 512 candidates per user) at full batch on the
    GPU; the oracle recomputes one user."""
    w = workloads.WORKLOADS["ranking_bf16"]
    inp = workloads.generate(w)
    attn = inp.attn
    lw = inp.layers[0]
    y = _gpu_layer(to_dev(inp.x, cuda_device), lw, attn, w, cuda_device)
    b = 3
    rows = rows_of(attn, [b])
    L = int(attn.lengths[b])
    ry = _oracle_layer(inp.x[torch.from_numpy(rows)], lw, attn, w, off=np.array([0, L]),
                       ts=attn.timestamps[torch.from_numpy(rows)], nt=attn.num_targets[b:b + 1])
    assert_bf16_close(y[torch.from_numpy(rows).to(cuda_device)], ry, what="ranking layer")
