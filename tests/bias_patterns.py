"""Seeded inputs that expose every relative-bias index the attention kernels compute.

Input construction only: no attention arithmetic lives here.

`patterns()` gives base sequences whose stamps drive each route the kernels take
through the temporal bucket and the positional clamp: unit gaps (differences
hit every 2^k - 1, 2^k and 2^k + 1 inside full tiles), gaps of 1023 and 1024
(1 + dt lands exactly on and one past powers of two), exponential gaps, gaps of
2^14 - 1 and 2^15 (differences near and past the 2^24 s rebasing limit),
epoch-scale stamps, block-wise descending stamps (negative differences),
equal stamps, geometrically growing gaps (rows spanning many buckets) and one
out-of-order stamp.

`readout_batch()` replicates each base sequence so that every visible pair is
read out on its own: with q = k = 0 the score of a pair is its bias alone, and
each copy gives one head a one-hot row of V (or of dO) on one block of d keys
(or queries) and zeros elsewhere, so every output element (O, or dV) holds the
weight of exactly one pair.

`readout_tables()` draws bias tables whose neighbouring entries differ by at
least 0.6 (positional) and 0.3 (temporal) and whose sums stay in [-0.7, 1.5],
where SiLU is increasing: an index off by one moves the pair's weight by far
more than bf16 rounding.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass
class Pattern:
    name: str
    stamps: np.ndarray       # int64 [L]
    n_targets: int = 0       # candidates at the end (used by the candidate variant)


def _blockwise_desc(L, rng, spread=1.3):
    out = []
    for b in range(0, L, 32):
        n = min(32, L - b)
        gaps = rng.exponential(300.0, n) * (spread ** np.arange(n))
        out.append(10**7 - 200_000 * (b // 32) + np.cumsum(gaps).astype(np.int64))
    return np.concatenate(out).astype(np.int64)


def patterns(seed=0, candidates=False):
    rng = np.random.default_rng(seed)
    j = lambda L: np.arange(L, dtype=np.int64)
    ps = [
        Pattern("unit_gaps", 1000 + j(1100), 100),
        Pattern("gap_1023", j(700) * 1023, 0),
        Pattern("gap_1024", j(900) * 1024, 64),
        Pattern("exp_300", np.floor(np.cumsum(rng.exponential(300.0, 1030))).astype(np.int64), 30),
        Pattern("gap_2p14_minus_1", j(1300) * 16383, 0),
        Pattern("gap_2p15", 77 + j(600) * 32768, 5),
        Pattern("epoch_exp_60", 1_700_000_000 + np.floor(np.cumsum(rng.exponential(60.0, 520))).astype(np.int64), 0),
        Pattern("blockwise_descending", _blockwise_desc(640, rng), 0),
        Pattern("equal", np.full(385, 5, dtype=np.int64), 1),
        Pattern("geometric", np.cumsum(np.floor(1.02 ** j(800))).astype(np.int64), 0),
    ]
    uns = np.floor(np.cumsum(rng.exponential(100.0, 450))).astype(np.int64)
    uns[200] = uns[199] - 1000  # one stamp out of order
    ps.append(Pattern("one_unsorted", uns, 0))
    if not candidates:
        for p in ps:
            p.n_targets = 0
    return ps


def readout_tables(lo, hi, nb, seed=1):
    rng = np.random.default_rng(seed)
    e = np.arange(hi - lo + 1)
    rab_pos = 0.2 + 1.0 * (e % 2) + 0.4 * rng.random(e.size)
    k = np.arange(nb)
    rab_time = -0.9 + 0.5 * (k % 2) + 0.2 * rng.random(nb)
    return (torch.from_numpy(rab_pos.astype(np.float32)), torch.from_numpy(rab_time.astype(np.float32)))


@dataclasses.dataclass
class Batch:
    seq_offsets: torch.Tensor   # int64 [B+1]
    timestamps: torch.Tensor    # int64 [T]
    num_targets: torch.Tensor | None
    lengths: list
    max_seq_len: int


def _batch(seqs):
    """seqs: list of (stamps, n_targets)."""
    lengths = [len(s) for s, _ in seqs]
    off = torch.from_numpy(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))
    ts = torch.from_numpy(np.concatenate([s for s, _ in seqs]).astype(np.int64))
    nts = [n for _, n in seqs]
    nt = torch.tensor(nts, dtype=torch.int32) if any(nts) else None
    return Batch(off, ts, nt, lengths, max(lengths))


def plain_batch(ps):
    """The base sequences once each."""
    return _batch([(p.stamps, p.n_targets) for p in ps])


def readout_batch(ps, H, d, which="v"):
    """Copies of every base sequence; copy c gives head h a one-hot block s = H c + h
    of d rows (keys for which="v", queries for which="dout"): row s d + m of that
    head holds e_m, every other row of the head zeros.  Returns the batch and the
    one-hot tensor [T, H, d] (bf16); q and k are zero."""
    seqs, onehots = [], []
    for p in ps:
        L = len(p.stamps)
        nblk = (L + d - 1) // d
        for c in range((nblk + H - 1) // H):
            oh = np.zeros((L, H, d), dtype=np.float32)
            for h in range(H):
                s = H * c + h
                if s >= nblk:
                    continue
                rows = np.arange(s * d, min(L, (s + 1) * d))
                oh[rows, h, rows - s * d] = 1.0
            seqs.append((p.stamps, p.n_targets))
            onehots.append(oh)
    b = _batch(seqs)
    return b, torch.from_numpy(np.concatenate(onehots)).to(torch.bfloat16)
