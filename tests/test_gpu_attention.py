"""GPU parity of the attention path against the CPU oracle (through the C ABI)."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import ops, workloads
from parity_utils import (assert_bf16_close, assert_f32_close, dev_attn, gpu_bwd, gpu_fwd,
                          attn_kwargs, sub_batch, to_dev)

pytestmark = pytest.mark.gpu


def _small(lengths, H=2, d=64, dtype=torch.bfloat16, nt=None, seed=0, epoch=0, lo=-300, hi=300,
           nb=32, n_scale=256, with_dout=True, gap=300.0):
    rng = np.random.default_rng(seed)
    return workloads.make_attn_inputs(rng, lengths, H, d, d, gap, lo, hi, nb, n_scale, dtype,
                                      num_targets=nt, with_dout=with_dout, epoch=epoch)


def _oracle_fwd(inp):
    return oracle.attn_fwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                           inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n)


def _oracle_bwd(inp):
    return oracle.attn_bwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                           inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, inp.dout)


# ---- scheduler and bias indices: exact -----------------------------------------

def expected_schedule(lengths, nts, tile, is_bwd, max_len):
    """The documented order: levels descending, sequences ascending inside a level."""
    nt = [0] * len(lengths) if nts is None else list(nts)
    ntiles = [(L + tile - 1) // tile if (L <= max_len and 0 <= n <= L) else 0
              for L, n in zip(lengths, nt)]
    items = []
    for level in reversed(range(max(1, (max_len + tile - 1) // tile))):
        for b, n in enumerate(ntiles):
            if n > level:
                items.append((b, n - 1 - level if is_bwd else level))
    return items


@pytest.mark.parametrize("is_bwd", [0, 1])
@pytest.mark.parametrize("case", ["mixed", "with_targets", "empty", "too_long"])
def test_schedule_exact(cuda_device, case, is_bwd):
    if case == "mixed":
        lengths, nts, max_len = [5, 0, 130, 64, 65, 1, 300], None, 300
    elif case == "with_targets":
        lengths, nts, max_len = [200, 90, 64], [30, 0, 64], 200
    elif case == "empty":
        lengths, nts, max_len = [0, 0, 0], None, 16
    else:
        lengths, nts, max_len = [10, 500, 20], None, 128
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    desc = ops.make_attn_desc(len(lengths), max_len, int(off[-1]), 1, 64, 64, ops.HSTU_BF16,
                              1.0, -8, 8, 4)
    nt_t = None if nts is None else torch.tensor(nts, dtype=torch.int32, device=cuda_device)
    items, count, hdr = ops.hstu_debug_schedule(desc, torch.from_numpy(off).to(cuda_device), nt_t,
                                                bool(is_bwd), 64)
    torch.cuda.synchronize()
    exp = expected_schedule(lengths, nts, 64, is_bwd, max_len)
    n = int(count.item())
    assert n == len(exp)
    assert [tuple(x) for x in items[:n].cpu().tolist()] == exp
    flag = int(hdr[0].item())
    assert flag == (4 if case == "too_long" else 0)


def test_bias_indices_exact(cuda_device):
    rng = np.random.default_rng(5)
    lengths = [40, 1, 300, 77]
    nts = [0, 0, 60, 7]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    # timestamps: epoch-scale, huge gaps around powers of two, equal and decreasing stamps
    ts = np.zeros(T, dtype=np.int64)
    for b in range(len(lengths)):
        s0, s1 = off[b], off[b + 1]
        base = [0, 1_700_000_000, (1 << 40) + 5, 123][b]
        gaps = rng.choice([0, 1, 2, 3, 7, 8, 1023, 1024, (1 << 20) - 1, 1 << 31, (1 << 33) + 1],
                          size=s1 - s0)
        ts[s0:s1] = base + np.cumsum(gaps)
    ts[off[3] + 5] = ts[off[3] + 4] - 9   # one out-of-order stamp
    pairs = []
    for b in range(len(lengths)):
        for _ in range(400):
            i, j = rng.integers(off[b], off[b + 1], size=2)
            pairs.append((i, j))
    pairs.append((0, off[1]))  # different sequences
    rows = np.array(pairs, dtype=np.int64)
    for lo, hi, nb in [(-128, 128, 64), (0, 127, 32), (-4096, 4096, 128), (-3, 5, 3)]:
        desc = ops.make_attn_desc(len(lengths), 300, T, 1, 64, 64, ops.HSTU_BF16, 1.0, lo, hi, nb)
        pos, bkt = ops.hstu_debug_bias_indices(
            desc, torch.from_numpy(off).to(cuda_device), torch.from_numpy(ts).to(cuda_device),
            torch.tensor(nts, dtype=torch.int32, device=cuda_device),
            torch.from_numpy(rows).to(cuda_device))
        pos, bkt = pos.cpu().numpy(), bkt.cpu().numpy()
        for e, (gi, gj) in enumerate(pairs):
            b = int(np.searchsorted(off, gi, side="right") - 1)
            if not (off[b] <= gj < off[b + 1]):
                assert pos[e] == -1 and bkt[e] == -1
                continue
            L, n = lengths[b], nts[b]
            i, j = gi - off[b], gj - off[b]
            hist = L - n
            pi, pj = min(i, hist), min(j, hist)
            assert pos[e] == oracle.pos_index(pi, pj, lo, hi)
            assert bkt[e] == oracle.time_bucket(ts[gi], ts[gj], nb)


def test_device_flag_reports_bad_offsets_without_fault(cuda_device):
    inp = _small([50, 70])
    d = dev_attn(inp, cuda_device)
    bad_off = torch.tensor([0, 80, 60], dtype=torch.int64, device=cuda_device)  # decreasing
    desc = ops.make_attn_desc(2, 128, 120, 2, 64, 64, ops.HSTU_BF16, inp.inv_n, inp.pos_lo,
                              inp.pos_hi, inp.rab_time.numel())
    ws = ops.alloc_workspace(ops.hstu_attn_workspace_size(desc, False), cuda_device)
    out = torch.zeros_like(d["v"])
    kw = dict(attn_kwargs(inp), max_seq_len=128)
    ops.hstu_attn_fwd(d["q"], d["k"], d["v"], bad_off, d["timestamps"], None, d["rab_pos"],
                      d["rab_time"], out=out, workspace=ws, **kw)
    st, bits = ops.hstu_check_device_flag(ws)
    assert st == 5 and bits & 2 and bits & 16
    # the valid first sequence was still computed
    ref = oracle.attn_fwd([0, 80], inp.timestamps[:80], None, inp.q[:80], inp.k[:80], inp.v[:80],
                          inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n)
    assert_bf16_close(out[:80], ref, what="valid sequence")
    # a correct call clears the flag
    ops.hstu_attn_fwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], None, d["rab_pos"],
                      d["rab_time"], out=out, workspace=ws, **kw)
    assert ops.hstu_check_device_flag(ws) == (0, 0)


def test_bounded_wait_runs_out_without_fault(cuda_device):
    # The timeout path of the pipeline waits, made to run on purpose with the
    # host-chosen test hook: the first CTA never loads its first key tile, its
    # waits give up after ~1 ms, the kernel ends, and the workspace flag
    # reports bit 32.  The next ordinary call on the same workspace is correct
    # and clears the flag.
    import ctypes
    inp = _small([700, 300, 513], H=2, d=64, seed=77)
    d = dev_attn(inp, cuda_device)
    desc = ops._attn_desc_from(d["q"], d["v"], d["seq_offsets"], inp.max_seq_len, inp.inv_n, inp.pos_lo,
                               inp.pos_hi, d["rab_pos"], d["rab_time"])
    desc.debug_checks = ops.HSTU_DEBUG_WAIT_TEST
    ws = ops.alloc_workspace(ops.hstu_attn_workspace_size(desc, False), cuda_device)
    out = torch.zeros_like(d["v"])
    lib = ops.load_library()
    p = lambda t: ctypes.c_void_p(0 if t is None else t.data_ptr())
    st = lib.hstu_attn_fwd(ctypes.byref(desc), p(d["q"]), p(d["k"]), p(d["v"]), p(d["seq_offsets"]),
                           p(d["timestamps"]), None, p(d["rab_pos"]), p(d["rab_time"]), p(out), p(ws),
                           ctypes.c_size_t(ws.numel()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    st, bits = ops.hstu_check_device_flag(ws)
    assert st == 5 and bits == 32
    ops.hstu_attn_fwd(d["q"], d["k"], d["v"], d["seq_offsets"], d["timestamps"], None, d["rab_pos"],
                      d["rab_time"], out=out, workspace=ws, **attn_kwargs(inp))
    assert ops.hstu_check_device_flag(ws) == (0, 0)
    assert_bf16_close(out, _oracle_fwd(inp), what="ordinary call after the timeout")


# ---- forward parity ------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
def test_fwd_small_ragged(cuda_device, d):
    # several tiles, ragged tails, an empty sequence, a single token, candidates
    inp = _small([1, 0, 63, 64, 65, 200, 129], H=2, d=d, nt=[0, 0, 5, 0, 64, 17, 1], seed=d)
    out = gpu_fwd(inp, cuda_device)
    assert_bf16_close(out, _oracle_fwd(inp), what=f"fwd d={d}")


def test_fwd_large_epoch_timestamps(cuda_device):
    inp = _small([150, 300], H=1, d=64, epoch=1_700_000_000, gap=5e6, nb=64, seed=9)
    assert_bf16_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what="epoch timestamps")


def test_fwd_all_empty(cuda_device):
    inp = _small([0, 0], H=2, d=64)
    out = gpu_fwd(inp, cuda_device)
    assert out.shape[0] == 0


def test_fwd_bwd_no_sequences(cuda_device):
    # B = 0, T = 0: every call is legal, launches nothing that touches rows, and
    # still zeroes the bias-table gradients
    dev = cuda_device
    z = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device=dev)
    off = torch.zeros(1, dtype=torch.int64, device=dev)
    ts = torch.zeros(0, dtype=torch.int64, device=dev)
    rp = torch.randn(17, device=dev)
    rt = torch.randn(8, device=dev)
    kw = dict(max_seq_len=0, inv_n=1.0, pos_lo=-8, pos_hi=8)
    out = ops.hstu_attn_fwd(z, z, z, off, ts, None, rp, rt, **kw)
    grads = (torch.empty_like(z), torch.empty_like(z), torch.empty_like(z),
             torch.full_like(rp, 7.0), torch.full_like(rt, 7.0))
    g = ops.hstu_attn_bwd(z, z, z, off, ts, None, rp, rt, z, grads=grads, **kw)
    torch.cuda.synchronize()
    assert out.shape == (0, 2, 64)
    assert not bool(g[3].any()) and not bool(g[4].any())


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_bwd_eight_heads(cuda_device, d):
    # more heads than the workloads use: the head index walks every per-head offset
    inp = _small([1, 130, 64, 257], H=8, d=d, nt=[0, 9, 0, 0], seed=70 + d)
    assert_bf16_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what=f"fwd H=8 d={d}")
    _check_bwd(gpu_bwd(inp, cuda_device), _oracle_bwd(inp), assert_bf16_close, f"bwd H=8 d={d}")


def test_fwd_attn_bf16_short_full(cuda_device):
    w = workloads.WORKLOADS["attn_bf16_short"]
    inp = workloads.generate(w)
    assert_bf16_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what="attn_bf16_short fwd")


def test_fwd_long_history_full_size_sampled(cuda_device):
    w = workloads.WORKLOADS["long_history_bf16"]
    inp = workloads.generate(w)
    out = gpu_fwd(inp, cuda_device)
    off = inp.seq_offsets.numpy()
    rng = np.random.default_rng(0)
    rows = []
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        rows += [s0, s0 + 1, s0 + 4095, s0 + 4097, s1 - 1] + list(rng.integers(s0, s1, size=3))
    rows = np.array(sorted(set(rows)), dtype=np.int64)
    ref = oracle.attn_fwd_rows(inp.seq_offsets, inp.timestamps, None, inp.q, inp.k, inp.v,
                               inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, rows)
    # the scale of the sampled rows stands in for the output's max-abs
    assert_bf16_close(out[torch.from_numpy(rows).to(cuda_device)], ref, what="long history rows")


def test_fwd_ranking_candidates(cuda_device):
    # ranking shapes at reduced batch: 2048 history + 512 candidates per user
    w = workloads.WORKLOADS["ranking_bf16"]
    rng = np.random.default_rng(w.seed)
    inp = workloads.make_attn_inputs(rng, [2560, 2560], 2, 128, 128, 120.0, -2560, 2560, 128, 2560,
                                     torch.bfloat16, num_targets=[512, 512])
    assert_bf16_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what="ranking fwd")


def test_fwd_f32(cuda_device):
    inp = _small([1, 70, 128, 33], H=2, d=32, dtype=torch.float32, nt=[0, 3, 0, 2], lo=0, hi=127,
                 n_scale=128, gap=60.0)
    assert_f32_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what="fwd f32")


# ---- backward parity -----------------------------------------------------------

def _check_bwd(gpu, ref, tol_fn, what):
    names = ["dq", "dk", "dv", "d_rab_pos", "d_rab_time"]
    for n, g, r in zip(names, gpu, ref):
        tol_fn(g, r, what=f"{what} {n}")


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_small_ragged(cuda_device, d):
    inp = _small([1, 0, 63, 64, 65, 200, 129], H=2, d=d, nt=[0, 0, 5, 0, 64, 17, 1], seed=10 + d)
    _check_bwd(gpu_bwd(inp, cuda_device), _oracle_bwd(inp), assert_bf16_close, f"bwd d={d}")


def test_bwd_attn_bf16_short_full(cuda_device):
    inp = workloads.generate(workloads.WORKLOADS["attn_bf16_short"])
    _check_bwd(gpu_bwd(inp, cuda_device), _oracle_bwd(inp), assert_bf16_close, "attn_bf16_short bwd")


def test_bwd_f32(cuda_device):
    inp = _small([1, 70, 128, 33], H=2, d=32, dtype=torch.float32, nt=[0, 3, 0, 2], lo=0, hi=127,
                 n_scale=128, gap=60.0, seed=3)
    _check_bwd(gpu_bwd(inp, cuda_device), _oracle_bwd(inp), assert_f32_close, "bwd f32")


def _blockwise_stamps(lengths, seed, spread):
    """Stamps sorted inside every aligned 32-token block but descending from
    block to block, so that visible pairs across blocks have negative
    differences while every warp's keys and queries are each sorted; `spread`
    makes the gaps inside a block grow geometrically (rows over many buckets)."""
    rng = np.random.default_rng(seed)
    out = []
    for L in lengths:
        for b in range(0, L, 32):
            n = min(32, L - b)
            gaps = rng.exponential(300.0, n) * (spread ** np.arange(n))
            out.append(10**7 - 200_000 * (b // 32) + np.cumsum(gaps).astype(np.int64))
    return torch.from_numpy(np.concatenate(out).astype(np.int64))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("spread", [1.0, 1.3])
def test_blockwise_sorted_stamps(cuda_device, d, spread):
    # fast-path classes with negative cross-block differences (bucket 0) and
    # rows spanning many buckets; forward and backward with the bias grads
    lengths = [200, 96, 130]
    inp = _small(lengths, H=2, d=d, seed=40 + d, nb=32)
    inp = dataclasses.replace(inp, timestamps=_blockwise_stamps(lengths, 41 + d, spread))
    assert_bf16_close(gpu_fwd(inp, cuda_device), _oracle_fwd(inp), what=f"fwd d={d} spread={spread}")
    _check_bwd(gpu_bwd(inp, cuda_device), _oracle_bwd(inp), assert_bf16_close, f"bwd d={d} spread={spread}")


def test_bwd_long_history_full_size_sampled(cuda_device):
    w = workloads.WORKLOADS["long_history_bf16"]
    inp = workloads.generate(w)
    dq, dk, dv, drp, drt = gpu_bwd(inp, cuda_device)
    off = inp.seq_offsets.numpy()
    rng = np.random.default_rng(1)
    qr, kr = [], []
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        qr += [s0, s0 + 4097, s1 - 1, int(rng.integers(s0, s1))]
        kr += [s0, s0 + 64, s1 - 129, s1 - 1, int(rng.integers(s0, s1))]
    qr, kr = np.array(qr, dtype=np.int64), np.array(kr, dtype=np.int64)
    rq, rk, rv = oracle.attn_bwd_rows(inp.seq_offsets, inp.timestamps, None, inp.q, inp.k, inp.v,
                                      inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n,
                                      inp.dout, qr, kr)
    dev = cuda_device
    assert_bf16_close(dq[torch.from_numpy(qr).to(dev)], rq, what="long dq rows")
    assert_bf16_close(dk[torch.from_numpy(kr).to(dev)], rk, what="long dk rows")
    assert_bf16_close(dv[torch.from_numpy(kr).to(dev)], rv, what="long dv rows")
    # both tables collect every dS once: their totals agree at any size
    tp, tt = float(drp.double().sum()), float(drt.double().sum())
    assert abs(tp - tt) <= 1e-3 * max(abs(tp), float(drp.abs().sum())), (tp, tt)


def test_bwd_long_history_full_size_tables_element_wise(cuda_device):
    """The full-size long-history backward (the bench's launch) with dout zero outside
    one sequence: every pair's score gradient is linear in dout_i, so the bias-table
    gradients hold that sequence's pairs alone and are compared element-wise with
    the oracle run on that sequence; every gradient row of the other sequences
    must be exactly zero."""
    w = workloads.WORKLOADS["long_history_bf16"]
    inp = workloads.generate(w)
    off = inp.seq_offsets.numpy()
    s = int(np.argmin(np.diff(off)))
    a, b = int(off[s]), int(off[s + 1])
    dout = torch.zeros_like(inp.dout)
    dout[a:b] = inp.dout[a:b]
    inp = dataclasses.replace(inp, dout=dout)
    dq, dk, dv, drp, drt = gpu_bwd(inp, cuda_device)
    ref = _oracle_bwd(sub_batch(inp, [s]))
    assert_bf16_close(drp, ref[3], what="full-size d_rab_pos")
    assert_bf16_close(drt, ref[4], what="full-size d_rab_time")
    for name, g, r in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
        assert_bf16_close(g[a:b], r, what=f"full-size {name} of the sequence")
        assert not bool(g[:a].any()) and not bool(g[b:].any()), f"{name} outside the sequence"


def test_bwd_long_history_bias_grads_one_sequence(cuda_device):
    # full bias-table gradients of one long sequence (clamps at +-4096)
    w = workloads.WORKLOADS["long_history_bf16"]
    rng = np.random.default_rng(w.seed + 77)
    inp = workloads.make_attn_inputs(rng, [4600], 4, 128, 128, 300.0, -4096, 4096, 128, 16384,
                                     torch.bfloat16, with_dout=True)
    g = gpu_bwd(inp, cuda_device)
    _check_bwd(g, _oracle_bwd(inp), assert_bf16_close, "long one-seq bwd")
