"""Exact checks of the relative-bias indices that the tcgen05 attention kernels compute
on their own fast paths (positional windows, the clamp folded into a constant,
the temporal bucket from the exponent of a rebased fp32 difference, one- and
two-bucket rows), through hstu_attn_fwd and hstu_attn_bwd.

The bias is the positional and temporal distance term of the DLRMv4 page's
"Model Architecture" section: rab_pos[clamp(p_i - p_j, lo, hi) - lo] +
rab_time[min(NB - 1, floor(log2(1 + max(t_i - t_j, 0))))].

- Single-pair readout (forward, and the backward's recomputed P through dV):
  with q = k = 0 a pair's score is its bias alone; V (or dO) one-hot on one
  block of keys (queries) per head and copy puts exactly one pair behind each
  output element, so an element equals SiLU(bias of that pair) (times 1/N = 1)
  up to the bf16 rounding of P.  The tables' neighbouring entries differ by at
  least 0.3, so one wrong index on one pair moves one element by more than
  0.05, against a tolerance of 6e-3 |ref| + 1e-3.
- Table-gradient histograms (backward): with q = k = 0, zero tables and
  v = dout = 1, every visible pair has the same score gradient d_v / (2N), so
  d_rab_pos[e] and d_rab_time[k] are H d_v / (2N) times the number of visible
  pairs on entry e / bucket k.  The counts come from the oracle
  (oracle.bias_pair_counts); every partial sum is an integer multiple of one
  power-of-two unit below 2^24 units, so the comparison is exact."""

import numpy as np
import pytest
import torch

import bias_patterns
import oracle
from hstu_sequential_transduction_b200 import flops, ops, workloads

pytestmark = pytest.mark.gpu

H = 2
# (pos_lo, pos_hi, num_time_buckets, candidates, local_window, global_window,
#  candidates at their own index, one table pair per head)
VARIANTS = {
    # clamp at 300 inside full tiles, 20 buckets (saturated by the 2^14 and 2^15 gaps)
    "causal": (-500, 300, 20, False, 0, 0, False, False),
    # candidates; lower clamp above 0 (distances 0..3 share an entry), upper at 129
    "candidates": (3, 129, 32, True, 0, 0, False, False),
    # semi-local windows, no clamp
    "windows": (0, 1400, 26, False, 300, 70, False, False),
    # both
    "candidates_windows": (-64, 2000, 24, True, 150, 33, False, False),
    # the same with candidates at their own index
    "candidates_own": (3, 129, 32, True, 0, 0, True, False),
    "candidates_windows_own": (-64, 2000, 24, True, 150, 33, True, False),
    # per-head tables
    "causal_per_head": (-500, 300, 20, False, 0, 0, False, True),
    "candidates_windows_own_per_head": (-64, 2000, 24, True, 150, 33, True, True),
}


def _tables(lo, hi, nb, seed, per_head):
    if not per_head:
        return bias_patterns.readout_tables(lo, hi, nb, seed=seed)
    ts = [bias_patterns.readout_tables(lo, hi, nb, seed=seed + 97 * h) for h in range(H)]
    return torch.stack([t[0] for t in ts]), torch.stack([t[1] for t in ts])


def _desc_kw(lo, hi, max_len, inv_n, lw, gw, own):
    return dict(max_seq_len=max_len, inv_n=inv_n, pos_lo=lo, pos_hi=hi, local_window=lw, global_window=gw,
                cand_own_index=own)


def _dev(t, dev):
    return None if t is None else t.to(dev).contiguous()


def _assert_readout(gpu, ref, what):
    g = gpu.detach().double().cpu().numpy()
    bad = np.abs(g - ref) > 6e-3 * np.abs(ref) + 1e-3
    if bad.any():
        idx = np.argwhere(bad)[:8]
        detail = ", ".join(f"{tuple(i)}: gpu {g[tuple(i)]:.5f} oracle {ref[tuple(i)]:.5f}" for i in idx)
        pytest.fail(f"{what}: {int(bad.sum())} of {bad.size} elements differ ({detail})")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_fwd_bias_single_pair_readout(cuda_device, d, variant):
    lo, hi, nb, cand, lw, gw, own, ph = VARIANTS[variant]
    ps = bias_patterns.patterns(seed=10, candidates=cand)
    b, v1 = bias_patterns.readout_batch(ps, H, d, "v")
    rp, rt = _tables(lo, hi, nb, 11, ph)
    T = b.timestamps.numel()
    z = torch.zeros((T, H, d), dtype=torch.bfloat16)
    dev = cuda_device
    zd = z.to(dev)
    out = ops.hstu_attn_fwd(zd, zd, v1.to(dev), _dev(b.seq_offsets, dev), _dev(b.timestamps, dev),
                            _dev(b.num_targets, dev), rp.to(dev), rt.to(dev),
                            **_desc_kw(lo, hi, b.max_seq_len, 1.0, lw, gw, own))
    torch.cuda.synchronize()
    ref = oracle.attn_fwd(b.seq_offsets, b.timestamps, b.num_targets, z, z, v1, rp, rt, lo, hi, 1.0,
                          local_window=lw, global_window=gw, cand_own_index=own)
    _assert_readout(out, ref, f"forward readout d={d} {variant}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_bwd_recomputed_bias_single_pair_readout(cuda_device, d, variant):
    # v = 0 and dO one-hot per query block: dV_j = P^T dO reads P of one pair per
    # element, while dP = 0 leaves every other gradient exactly zero
    lo, hi, nb, cand, lw, gw, own, ph = VARIANTS[variant]
    ps = bias_patterns.patterns(seed=20, candidates=cand)
    b, do1 = bias_patterns.readout_batch(ps, H, d, "dout")
    rp, rt = _tables(lo, hi, nb, 21, ph)
    T = b.timestamps.numel()
    z = torch.zeros((T, H, d), dtype=torch.bfloat16)
    dev = cuda_device
    zd = z.to(dev)
    dq, dk, dv, drp, drt = ops.hstu_attn_bwd(zd, zd, zd, _dev(b.seq_offsets, dev), _dev(b.timestamps, dev),
                                             _dev(b.num_targets, dev), rp.to(dev), rt.to(dev), do1.to(dev),
                                             **_desc_kw(lo, hi, b.max_seq_len, 1.0, lw, gw, own))
    torch.cuda.synchronize()
    _, _, rdv, _, _ = oracle.attn_bwd(b.seq_offsets, b.timestamps, b.num_targets, z, z, z, rp, rt, lo, hi, 1.0,
                                      do1, local_window=lw, global_window=gw, cand_own_index=own)
    _assert_readout(dv, rdv, f"backward dV readout d={d} {variant}")
    for name, t in (("dq", dq), ("dk", dk), ("d_rab_pos", drp), ("d_rab_time", drt)):
        assert not bool(t.any()), f"{name} should be exactly zero"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_bwd_bias_grad_histogram_exact(cuda_device, d, variant):
    lo, hi, nb, cand, lw, gw, own, ph = VARIANTS[variant]
    ps = bias_patterns.patterns(seed=30, candidates=cand)
    b = bias_patterns.plain_batch(ps)
    T = b.timestamps.numel()
    inv_n = 1.0 / 1024
    dev = cuda_device
    zd = torch.zeros((T, H, d), dtype=torch.bfloat16, device=dev)
    one = torch.ones((T, H, d), dtype=torch.bfloat16, device=dev)
    rows = (H,) if ph else ()
    zp = torch.zeros(rows + (hi - lo + 1,), dtype=torch.float32, device=dev)
    zt = torch.zeros(rows + (nb,), dtype=torch.float32, device=dev)
    _, _, _, drp, drt = ops.hstu_attn_bwd(zd, zd, one, _dev(b.seq_offsets, dev), _dev(b.timestamps, dev),
                                          _dev(b.num_targets, dev), zp, zt, one,
                                          **_desc_kw(lo, hi, b.max_seq_len, inv_n, lw, gw, own))
    torch.cuda.synchronize()
    pc, tc = oracle.bias_pair_counts(b.seq_offsets, b.timestamps, b.num_targets, lo, hi, nb, lw, gw,
                                     cand_own_index=own)
    # each head's pairs land in its own row with per-head tables, in the one row otherwise
    unit = (1 if ph else H) * d * 0.5 * inv_n
    assert pc.sum() * H < 2**24  # every partial sum exact in fp32
    if ph:
        pc, tc = np.tile(pc, (H, 1)), np.tile(tc, (H, 1))
    got_p = drp.cpu().double().numpy().reshape(pc.shape)
    got_t = drt.cpu().double().numpy().reshape(tc.shape)
    assert tuple(drp.shape) == tuple(zp.shape) and tuple(drt.shape) == tuple(zt.shape)
    got_p, got_t, pc, tc = got_p.reshape(-1), got_t.reshape(-1), pc.reshape(-1), tc.reshape(-1)
    bad_p = np.flatnonzero(got_p != pc * unit)
    bad_t = np.flatnonzero(got_t != tc * unit)
    npos = hi - lo + 1
    assert bad_p.size == 0, f"rab_pos entries {bad_p[:10] % npos + lo} (distance; head {bad_p[:10] // npos}): " \
                            f"gpu {got_p[bad_p[:10]] / unit} pairs vs {pc[bad_p[:10]]}"
    assert bad_t.size == 0, f"rab_time buckets {bad_t[:10]}: gpu {got_t[bad_t[:10]] / unit} pairs vs {tc[bad_t[:10]]}"


def test_bwd_bias_grad_histogram_long_history_full_size(cuda_device):
    """The long-history workload at full size (8 sequences of U[8192, 16384] tokens,
    4 heads of 128, positions clamped at 4096, 128 buckets) with q = k = 0, zero
    tables and v = dout = 1: every entry's gradient is the pair count times
    H d / (2N).  Entries holding fewer than 2^24 / H pairs are compared exactly;
    the few larger ones (the clamped distance, the populated high buckets) at
    1e-4 relative (fp32 addition of up to ~10^8 equal terms)."""
    w = workloads.WORKLOADS["long_history_bf16"]
    inp = workloads.generate(w)
    dev = cuda_device
    T, Hh, d = inp.total_tokens, w.num_heads, w.d_qk
    zd = torch.zeros((T, Hh, d), dtype=torch.bfloat16, device=dev)
    one = torch.ones((T, Hh, d), dtype=torch.bfloat16, device=dev)
    zp = torch.zeros(inp.pos_hi - inp.pos_lo + 1, dtype=torch.float32, device=dev)
    nb = inp.rab_time.numel()
    zt = torch.zeros(nb, dtype=torch.float32, device=dev)
    _, _, _, drp, drt = ops.hstu_attn_bwd(zd, zd, one, inp.seq_offsets.to(dev), inp.timestamps.to(dev), None,
                                          zp, zt, one, max_seq_len=inp.max_seq_len, inv_n=inp.inv_n,
                                          pos_lo=inp.pos_lo, pos_hi=inp.pos_hi)
    torch.cuda.synchronize()
    pc, tc = oracle.bias_pair_counts(inp.seq_offsets, inp.timestamps, None, inp.pos_lo, inp.pos_hi, nb)
    assert pc.sum() == tc.sum() == flops.attn_pairs(inp.lengths, None)
    unit = Hh * d * 0.5 * inp.inv_n
    for name, got, cnt in (("d_rab_pos", drp, pc), ("d_rab_time", drt, tc)):
        g = got.cpu().double().numpy()
        e = cnt * unit
        small = cnt * Hh < 2**24
        bad = np.flatnonzero(small & (g != e))
        assert bad.size == 0, f"{name} entries {bad[:10]}: gpu {g[bad[:10]] / unit} pairs vs {cnt[bad[:10]]}"
        big = ~small
        if big.any():
            rel = np.abs(g[big] - e[big]) / e[big]
            assert rel.max() <= 1e-4, f"{name} large entries: max relative error {rel.max():.2e}"
