"""Shared helpers of the GPU parity tests (inputs to device, error measures)."""

from __future__ import annotations

import numpy as np
import torch

from hstu_sequential_transduction_b200 import ops

# bf16 workloads: max |gpu - oracle| <= 2e-2 * max |oracle| per tensor.
BF16_TOL = 2e-2
# fp32 workloads: |gpu - oracle| <= 1e-4 * max(|oracle|, 1e-2 * max |oracle|) elementwise.
F32_TOL = 1e-4


def to_dev(t, dev):
    return None if t is None else t.to(dev).contiguous()


def np64(t):
    return t.detach().float().cpu().double().numpy() if t.dtype != torch.float64 else t.cpu().numpy()


def maxabs_rel_err(gpu, ref):
    g, r = np64(gpu) if torch.is_tensor(gpu) else gpu, ref
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    err = float(np.max(np.abs(g - r))) if r.size else 0.0
    return err / scale if scale > 0 else err


def assert_bf16_close(gpu, ref, tol=BF16_TOL, what=""):
    e = maxabs_rel_err(gpu, ref)
    assert e <= tol, f"{what}: max-abs-relative error {e:.3e} > {tol}"
    return e


def assert_f32_close(gpu, ref, tol=F32_TOL, what=""):
    g = np64(gpu) if torch.is_tensor(gpu) else gpu
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    denom = np.maximum(np.abs(ref), 1e-2 * scale)
    denom = np.where(denom > 0, denom, 1.0)
    e = float(np.max(np.abs(g - ref) / denom)) if ref.size else 0.0
    assert e <= tol, f"{what}: max relative error {e:.3e} > {tol}"
    return e


def attn_kwargs(inp):
    return dict(max_seq_len=inp.max_seq_len, inv_n=inp.inv_n, pos_lo=inp.pos_lo, pos_hi=inp.pos_hi)


def dev_attn(inp, dev):
    """The attention tensors of a workloads.AttnInputs on the device."""
    return dict(q=to_dev(inp.q, dev), k=to_dev(inp.k, dev), v=to_dev(inp.v, dev),
                seq_offsets=to_dev(inp.seq_offsets, dev), timestamps=to_dev(inp.timestamps, dev),
                num_targets=to_dev(inp.num_targets, dev), rab_pos=to_dev(inp.rab_pos, dev),
                rab_time=to_dev(inp.rab_time, dev),
                dout=to_dev(inp.dout, dev) if inp.dout is not None else None)


def gpu_fwd(inp, dev, **windows):
    d = dev_attn(inp, dev)
    out = ops.hstu_attn_fwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                            d["num_targets"], d["rab_pos"], d["rab_time"], **attn_kwargs(inp), **windows)
    torch.cuda.synchronize()
    return out


def gpu_bwd(inp, dev, **windows):
    d = dev_attn(inp, dev)
    g = ops.hstu_attn_bwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], d["num_targets"],
                          d["rab_pos"], d["rab_time"], d["dout"], **attn_kwargs(inp), **windows)
    torch.cuda.synchronize()
    return g


def sub_batch(inp, seqs):
    """A workloads.AttnInputs holding only sequences `seqs` (values copied)."""
    import dataclasses
    off = inp.seq_offsets.numpy()
    sl = [slice(int(off[b]), int(off[b + 1])) for b in seqs]
    lengths = [s.stop - s.start for s in sl]
    new_off = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))
    cat = lambda t: None if t is None else torch.cat([t[s] for s in sl])
    nt = None if inp.num_targets is None else inp.num_targets[list(seqs)].clone()
    return dataclasses.replace(inp, seq_offsets=new_off, timestamps=cat(inp.timestamps),
                               num_targets=nt, q=cat(inp.q), k=cat(inp.k), v=cat(inp.v),
                               dout=cat(inp.dout), max_seq_len=max(lengths) if lengths else 0)


def rows_of(inp, seqs):
    off = inp.seq_offsets.numpy()
    return np.concatenate([np.arange(off[b], off[b + 1]) for b in seqs]).astype(np.int64)
