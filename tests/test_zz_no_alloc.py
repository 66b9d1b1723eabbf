"""The no-allocation forward entry point (for callers that cannot allocate
device memory, e.g. a plugin whose host framework owns every allocation).

It runs the same kernels as hstu_attn_fwd, only with its scheduler scratch in a
static device array, so on two calls in a row with different inputs (the
static scratch is shared and keeps the previous call's contents) its output
must be bit-identical to hstu_attn_fwd's with a caller workspace; the first
case is also held to the oracle at the bf16 tolerance.  This file is collected
last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import assert_bf16_close, attn_kwargs, dev_attn


def _inputs(seed, lengths, nt):
    rng = np.random.default_rng(seed)
    return workloads.make_attn_inputs(rng, lengths, 2, 64, 64, 300.0, -512, 512, 64, 1024,
                                      torch.bfloat16, num_targets=nt)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_two_calls(cuda_device):
    cases = [_inputs(1, [300, 1, 0, 129, 64], [0, 0, 0, 9, 64]), _inputs(2, [1000, 77], None)]
    outs = []
    for inp in cases:
        d = dev_attn(inp, cuda_device)
        out = torch.empty_like(d["v"])
        ops.hstu_attn_fwd_noalloc(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                                  d["num_targets"], d["rab_pos"], d["rab_time"], out,
                                  **attn_kwargs(inp))
        outs.append((inp, d, out))
    torch.cuda.synchronize()
    for inp, d, out in outs:
        ref = ops.hstu_attn_fwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"],
                                d["num_targets"], d["rab_pos"], d["rab_time"], **attn_kwargs(inp))
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    inp, _, out = outs[0]
    ref = oracle.attn_fwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                          inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n)
    assert_bf16_close(out, ref, what="no-allocation forward against the oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = ops.load_library()
    # 64 * 70000 tokens need more than 65536 work items
    desc = ops.make_attn_desc(1, 1 << 20, 64 * 70000, 1, 64, 64, ops.HSTU_BF16, 1.0, -8, 8, 4)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check fails first
    st = lib.hstu_attn_fwd_noalloc(ctypes.byref(desc), fake, fake, fake, fake, fake, None, fake,
                                   fake, fake, None)
    assert st == 2
