"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test states what fixes the expected value: the hand-worked example in
tests/golden (derived from the definition on the "HSTU Architecture" and
"Model Architecture" sections), a dense formulation written independently
with numpy, torch float64 autograd, central finite differences, invariants,
exhaustive integer checks and the DLRMv4 page's Table 7 cost formulas.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from hstu_sequential_transduction_b200 import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line or "=" not in line:
                continue
            key, val = [s.strip() for s in line.split("=", 1)]
            vals[key] = [float(x) for x in val.split()]
    return vals


# ---- independent dense formulation (numpy) ---------------------------------

def dense_bias_and_mask(L, n_t, t, lo, hi, rab_pos, rab_time):
    hist = L - n_t
    idx = np.arange(L)
    p = np.where(idx < hist, idx, hist)
    rel = np.clip(p[:, None] - p[None, :], lo, hi) - lo
    nb = len(rab_time)
    dt = np.maximum(t[:, None].astype(object) - t[None, :].astype(object), 0)
    bkt = np.vectorize(lambda x: min(nb - 1, (int(x) + 1).bit_length() - 1), otypes=[np.int64])(dt)
    bias = np.asarray(rab_pos)[rel] + np.asarray(rab_time)[bkt]
    I, J = idx[:, None], idx[None, :]
    vis = np.where(I < hist, J <= I, (J < hist) | (J == I))
    return bias, vis


def dense_fwd(off, ts, nt, q, k, v, rab_pos, rab_time, lo, hi, inv_n):
    T, H, dv = v.shape
    out = np.zeros((T, H, dv))
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        bias, vis = dense_bias_and_mask(L, n_t, ts[s0:s1], lo, hi, rab_pos, rab_time)
        S = np.einsum("ihc,jhc->hij", q[s0:s1], k[s0:s1]) + bias[None]
        P = S / (1.0 + np.exp(-S)) * inv_n * vis[None]
        out[s0:s1] = np.einsum("hij,jhc->ihc", P, v[s0:s1])
    return out


def rand_case(rng, lengths, H=2, dqk=3, dv=2, nt=None, lo=-3, hi=4, nb=5, gap=3.0, inv_n=0.5):
    lengths = np.asarray(lengths)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    ts = []
    for b, L in enumerate(lengths):
        ts.append(np.cumsum(rng.integers(0, int(2 * gap) + 1, size=L)))
    ts = np.concatenate(ts).astype(np.int64) if T else np.zeros(0, np.int64)
    q = rng.standard_normal((T, H, dqk))
    k = rng.standard_normal((T, H, dqk))
    v = rng.standard_normal((T, H, dv))
    rp = rng.standard_normal(hi - lo + 1) * 0.3
    rt = rng.standard_normal(nb) * 0.3
    nta = None if nt is None else np.asarray(nt, dtype=np.int32)
    return dict(seq_offsets=off, timestamps=ts, num_targets=nta, q=q, k=k, v=v, rab_pos=rp,
                rab_time=rt, pos_lo=lo, pos_hi=hi, inv_n=inv_n)


def ofwd(c, **kw):
    d = dict(c)
    d.update(kw)
    return oracle.attn_fwd(d["seq_offsets"], d["timestamps"], d["num_targets"], d["q"], d["k"],
                           d["v"], d["rab_pos"], d["rab_time"], d["pos_lo"], d["pos_hi"], d["inv_n"])


def dfwd(c):
    return dense_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                     c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])


# ---- 1. hand-worked example -------------------------------------------------

def test_hand_worked_three_tokens():
    g = _parse_golden("hand_3token.txt")
    q = np.array(g["q"]).reshape(3, 1, 1)
    k = np.array(g["k"]).reshape(3, 1, 1)
    v = np.array(g["v"]).reshape(3, 1, 1)
    t = np.array(g["t"], dtype=np.int64)
    out = oracle.attn_fwd([0, 3], t, None, q, k, v, g["rab_pos"], g["rab_time"],
                          int(g["pos_lo"][0]), int(g["pos_hi"][0]), 1.0 / g["N"][0])
    np.testing.assert_allclose(out.reshape(3), g["O"], rtol=0, atol=g["tolerance"][0])


def test_hand_worked_buckets():
    # the example's buckets: dt = 0, 3, 7, 10 -> 0, 2, 3, 3 (capped at 3)
    assert [oracle.time_bucket(dt, 0, 4) for dt in (0, 3, 7, 10)] == [0, 2, 3, 3]


# ---- 2. brute force: dense formulation --------------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_loops_match_dense(seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(0, 9, size=4)
    nt = None
    if seed % 2:
        nt = [int(rng.integers(0, L + 1)) for L in lengths]
    c = rand_case(rng, lengths, nt=nt, lo=-2 - seed, hi=3, nb=3 + seed)
    np.testing.assert_allclose(ofwd(c), dfwd(c), rtol=0, atol=1e-12)


def test_rows_variant_matches_full():
    rng = np.random.default_rng(7)
    c = rand_case(rng, [5, 0, 7, 3], nt=[1, 0, 2, 0])
    full = ofwd(c)
    rows = np.array([0, 4, 5, 9, 11, 14])
    part = oracle.attn_fwd_rows(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"],
                                c["v"], c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"],
                                c["inv_n"], rows)
    np.testing.assert_array_equal(part, full[rows])


# ---- 3. invariants -------------------------------------------------------------

def test_causality_future_tokens_do_not_change_past_rows():
    rng = np.random.default_rng(11)
    c = rand_case(rng, [9])
    base = ofwd(c)
    i0 = 4
    c2 = dict(c)
    for key in ("q", "k", "v"):
        a = c[key].copy()
        a[i0 + 1:] = rng.standard_normal(a[i0 + 1:].shape)
        c2[key] = a
    t = c["timestamps"].copy()
    t[i0 + 1:] += 1000
    c2["timestamps"] = t
    out = ofwd(c2)
    np.testing.assert_array_equal(out[: i0 + 1], base[: i0 + 1])
    assert not np.array_equal(out[i0 + 1:], base[i0 + 1:])


def test_sequences_are_independent():
    rng = np.random.default_rng(12)
    lengths = [4, 6, 3]
    c = rand_case(rng, lengths)
    base = ofwd(c)
    off = c["seq_offsets"]
    for b in range(3):
        s0, s1 = off[b], off[b + 1]
        alone = dict(c, seq_offsets=np.array([0, s1 - s0]), timestamps=c["timestamps"][s0:s1],
                     q=c["q"][s0:s1], k=c["k"][s0:s1], v=c["v"][s0:s1])
        np.testing.assert_array_equal(ofwd(alone), base[s0:s1])
    # permuted batch: [2, 0, 1]
    perm = [2, 0, 1]
    sl = [slice(off[b], off[b + 1]) for b in perm]
    pc = dict(c, seq_offsets=np.concatenate([[0], np.cumsum([lengths[b] for b in perm])]),
              timestamps=np.concatenate([c["timestamps"][s] for s in sl]),
              q=np.concatenate([c["q"][s] for s in sl]), k=np.concatenate([c["k"][s] for s in sl]),
              v=np.concatenate([c["v"][s] for s in sl]))
    np.testing.assert_array_equal(ofwd(pc), np.concatenate([base[s] for s in sl]))


def test_zero_bias_is_plain_silu_attention():
    rng = np.random.default_rng(13)
    c = rand_case(rng, [7])
    c = dict(c, rab_pos=np.zeros_like(c["rab_pos"]), rab_time=np.zeros_like(c["rab_time"]))
    q, k, v = c["q"][:, 0], c["k"][:, 0], c["v"][:, 0]
    S = q @ k.T
    P = S / (1 + np.exp(-S)) * c["inv_n"] * np.tril(np.ones((7, 7)))
    np.testing.assert_allclose(ofwd(c)[:, 0], P @ v, rtol=0, atol=1e-12)


def test_linear_in_v():
    rng = np.random.default_rng(14)
    c = rand_case(rng, [6, 5])
    v2 = rng.standard_normal(c["v"].shape)
    lhs = ofwd(c, v=2.0 * c["v"] - 3.0 * v2)
    rhs = 2.0 * ofwd(c) - 3.0 * ofwd(c, v=v2)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-11)


def test_constant_bias_shift_moves_between_tables():
    rng = np.random.default_rng(15)
    c = rand_case(rng, [8, 4], nt=[2, 1])
    a = ofwd(c, rab_pos=c["rab_pos"] + 0.375)
    b = ofwd(c, rab_time=c["rab_time"] + 0.375)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


# ---- 4. special cases ---------------------------------------------------------

def test_single_token_closed_form():
    rng = np.random.default_rng(16)
    c = rand_case(rng, [1], H=1, dqk=4, dv=3)
    s = float(c["q"][0, 0] @ c["k"][0, 0]) + c["rab_pos"][0 - c["pos_lo"]] + c["rab_time"][0]
    expect = s / (1 + np.exp(-s)) * c["inv_n"] * c["v"][0, 0]
    np.testing.assert_allclose(ofwd(c)[0, 0], expect, rtol=0, atol=1e-14)


def test_zero_qk_and_bias_gives_zero():
    rng = np.random.default_rng(17)
    c = rand_case(rng, [5, 3])
    out = ofwd(c, q=np.zeros_like(c["q"]), k=np.zeros_like(c["k"]),
               rab_pos=np.zeros_like(c["rab_pos"]), rab_time=np.zeros_like(c["rab_time"]))
    assert np.all(out == 0.0)


def test_empty_batch_and_empty_sequences():
    rng = np.random.default_rng(18)
    c = rand_case(rng, [0, 0, 3, 0])
    np.testing.assert_allclose(ofwd(c), dfwd(c), rtol=0, atol=1e-12)


def test_candidate_rows_by_hand():
    # 2 history tokens + 2 candidates; q=k=0 so s = pos bias + time bias only.
    # candidate rows sit at position 2: they see j=0 (dist 2), j=1 (dist 1),
    # themselves (dist 0), and not the other candidate.
    L, nt = 4, 2
    q = np.zeros((L, 1, 1))
    k = np.zeros((L, 1, 1))
    v = np.array([1.0, 10.0, 100.0, 1000.0]).reshape(L, 1, 1)
    t = np.array([0, 0, 0, 0], dtype=np.int64)
    rp = np.array([0.5, 1.0, 2.0])  # distances 0, 1, 2 (lo=0, hi=2)
    rt = np.array([0.0])
    out = oracle.attn_fwd([0, L], t, [nt], q, k, v, rp, rt, 0, 2, 1.0).reshape(L)
    sl = lambda x: x / (1 + np.exp(-x))
    assert out[2] == pytest.approx(sl(2.0) * 1 + sl(1.0) * 10 + sl(0.5) * 100, abs=1e-12)
    assert out[3] == pytest.approx(sl(2.0) * 1 + sl(1.0) * 10 + sl(0.5) * 1000, abs=1e-12)
    assert out[1] == pytest.approx(sl(1.0) * 1 + sl(0.5) * 10, abs=1e-12)


# ---- 5. gradients: torch float64 autograd and finite differences -------------

def _torch_dense_loss(c, dout):
    off, nt = c["seq_offsets"], c["num_targets"]
    q = torch.tensor(c["q"], requires_grad=True)
    k = torch.tensor(c["k"], requires_grad=True)
    v = torch.tensor(c["v"], requires_grad=True)
    rp = torch.tensor(c["rab_pos"], requires_grad=True)
    rt = torch.tensor(c["rab_time"], requires_grad=True)
    loss = 0.0
    lo, hi = c["pos_lo"], c["pos_hi"]
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        hist = L - n_t
        idx = np.arange(L)
        p = np.where(idx < hist, idx, hist)
        rel = torch.tensor(np.clip(p[:, None] - p[None, :], lo, hi) - lo)
        ts = c["timestamps"][s0:s1]
        bkt = torch.tensor([[min(len(c["rab_time"]) - 1, (int(max(ts[i] - ts[j], 0)) + 1).bit_length() - 1)
                             for j in range(L)] for i in range(L)])
        I, J = idx[:, None], idx[None, :]
        vis = torch.tensor(np.where(I < hist, J <= I, (J < hist) | (J == I)), dtype=torch.float64)
        S = torch.einsum("ihc,jhc->hij", q[s0:s1], k[s0:s1]) + (rp[rel] + rt[bkt])[None]
        P = torch.nn.functional.silu(S) * c["inv_n"] * vis[None]
        O = torch.einsum("hij,jhc->ihc", P, v[s0:s1])
        loss = loss + (O * torch.tensor(dout[s0:s1])).sum()
    loss.backward()
    return [x.grad.numpy() for x in (q, k, v, rp, rt)]


def obwd(c, dout):
    return oracle.attn_bwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"],
                           c["v"], c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"],
                           c["inv_n"], dout)


@pytest.mark.parametrize("seed", range(4))
def test_bwd_matches_torch_autograd(seed):
    rng = np.random.default_rng(100 + seed)
    lengths = rng.integers(1, 8, size=3)
    nt = [int(rng.integers(0, L)) for L in lengths] if seed % 2 else None
    c = rand_case(rng, lengths, nt=nt)
    dout = rng.standard_normal(c["v"].shape)
    ours = obwd(c, dout)
    ref = _torch_dense_loss(c, dout)
    for a, b in zip(ours, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_bwd_central_finite_differences():
    rng = np.random.default_rng(200)
    c = rand_case(rng, [4, 3], H=2, dqk=2, dv=2, nt=[1, 0])
    dout = rng.standard_normal(c["v"].shape)
    grads = dict(zip(["q", "k", "v", "rab_pos", "rab_time"], obwd(c, dout)))
    h = 1e-5
    for key, g in grads.items():
        flat = c[key].reshape(-1)
        for e in range(flat.size):
            plus, minus = flat.copy(), flat.copy()
            plus[e] += h
            minus[e] -= h
            fp = np.sum(ofwd(c, **{key: plus.reshape(c[key].shape)}) * dout)
            fm = np.sum(ofwd(c, **{key: minus.reshape(c[key].shape)}) * dout)
            assert abs((fp - fm) / (2 * h) - g.reshape(-1)[e]) < 1e-7, (key, e)


def test_bwd_rows_match_full():
    rng = np.random.default_rng(201)
    c = rand_case(rng, [6, 4, 5], nt=[0, 1, 2])
    dout = rng.standard_normal(c["v"].shape)
    dq, dk, dv, _, _ = obwd(c, dout)
    qr, kr = np.array([0, 5, 7, 14]), np.array([1, 6, 9, 10, 14])
    pq, pk, pv = oracle.attn_bwd_rows(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"],
                                      c["k"], c["v"], c["rab_pos"], c["rab_time"], c["pos_lo"],
                                      c["pos_hi"], c["inv_n"], dout, qr, kr)
    np.testing.assert_allclose(pq, dq[qr], rtol=0, atol=1e-12)
    np.testing.assert_allclose(pk, dk[kr], rtol=0, atol=1e-12)
    np.testing.assert_allclose(pv, dv[kr], rtol=0, atol=1e-12)


def test_bias_grad_tables_sum_to_the_same_total():
    rng = np.random.default_rng(202)
    c = rand_case(rng, [7, 5])
    dout = rng.standard_normal(c["v"].shape)
    _, _, _, drp, drt = obwd(c, dout)
    assert drp.sum() == pytest.approx(drt.sum(), abs=1e-12)


# ---- 6. bucket and position functions: exhaustive integer checks ---------------

def _bucket_by_powers(dt, nb):
    # largest b with 2**b <= 1 + max(dt, 0), capped at nb - 1
    x = 1 + max(dt, 0)
    b = 0
    while (1 << (b + 1)) <= x:
        b += 1
    return min(b, nb - 1)


def test_bucket_exhaustive_small_range():
    lib = oracle._load()
    for dt in range(0, 1 << 20, 1):
        if dt < 4096 or dt % 97 == 0 or (dt & (dt + 1)) == 0 or (dt & (dt - 1)) == 0:
            assert lib.oracle_time_bucket(dt, 0, 128) == _bucket_by_powers(dt, 128)


def test_bucket_numpy_exhaustive_2_20():
    # the whole [0, 2^20] range against powers-of-two boundaries (vectorised)
    dt = np.arange(0, (1 << 20) + 1, dtype=np.int64)
    expect = np.searchsorted(1 << np.arange(0, 40, dtype=np.int64), dt + 1, side="right") - 1
    lib = oracle._load()
    sample = dt[:: 1 << 10]
    got = np.array([lib.oracle_time_bucket(int(x), 0, 64) for x in sample])
    np.testing.assert_array_equal(got, np.minimum(expect[:: 1 << 10], 63))


def test_bucket_powers_of_two_and_large_epochs():
    for e in range(0, 63):
        for d in (-1, 0, 1):
            dt = (1 << e) + d - 1
            if dt < 0:
                continue
            for base in (0, 1_700_000_000, (1 << 40) + 3):
                assert oracle.time_bucket(base + dt, base, 128) == _bucket_by_powers(dt, 128)
                assert oracle.time_bucket(base + dt, base, 16) == _bucket_by_powers(dt, 16)
    assert oracle.time_bucket(5, 9, 32) == 0   # negative elapsed time clamps to 0


def test_pos_index_clamps():
    assert oracle.pos_index(10, 3, -4, 4) == 8
    assert oracle.pos_index(3, 10, -4, 4) == 0
    assert oracle.pos_index(5, 5, -4, 4) == 4
    assert oracle.pos_index(127, 0, 0, 127) == 127
    assert oracle.pos_index(0, 1, 0, 127) == 0


def test_visibility_rule():
    # history rows: j <= i; candidate rows: all history and themselves
    L, nt = 6, 2
    vis = [[oracle.visible(i, j, L, nt) for j in range(L)] for i in range(L)]
    assert vis[3] == [True, True, True, True, False, False]
    assert vis[4] == [True, True, True, True, True, False]
    assert vis[5] == [True, True, True, True, False, True]


# ---- 7. FLOP accounting: the DLRMv4 page's Table 7 ---------------------------

def test_cost_table_reproduces_published_figures():
    # Table 6 symbols: B=1024, L=3 layers, h=4, d_qk=d_v=128, D=512, S=4096
    B, layers, h, d, D, S = 1024, 3, 4, 128, 512, 4096
    pairs_lower_triangle = B * S * S / 2            # the page's S^2/2 per sequence
    attn = layers * (flops.attn_fwd_flops(pairs_lower_triangle, h, d, d)
                     + flops.attn_bwd_flops(pairs_lower_triangle, h, d, d))
    assert round(attn / 1e12, 2) == 184.72
    uvqk = layers * 3 * flops.f1_flops(B * S, D, h, d, d)
    assert round(uvqk / 1e12, 2) == 79.16
    outp = layers * 3 * flops.f2_flops(B * S, D, h, d, width_factor=3)
    assert round(outp / 1e12, 2) == 59.37
    assert round((attn + uvqk + outp) / 1e12, 2) == 323.26
    # backward is 2.5x forward: the "factor 3.5" for fwd+bwd
    assert flops.attn_bwd_flops(1, h, d, d) == 2.5 * flops.attn_fwd_flops(1, h, d, d)
    # projections: the table's rows count forward + backward as 3x the forward GEMM
    f1, f2 = flops.f1_flops(B * S, D, h, d, d), flops.f2_flops(B * S, D, h, d)
    assert flops.layer_bwd_gemm_flops(B * S, D, h, d, d) == 2 * (f1 + f2)


def test_pair_counter_by_brute_force():
    for L, nt in [(1, 0), (5, 0), (9, 3), (6, 6), (4096, 0), (2560, 512)]:
        if L <= 16:
            brute = sum(oracle.visible(i, j, L, nt) for i in range(L) for j in range(L))
            assert flops.attn_pairs_per_seq(L, nt) == brute
    assert flops.attn_pairs_per_seq(4096) == 4096 * 4097 // 2
    assert flops.attn_pairs([3, 0, 2], [1, 0, 0]) == (3 + 3) + 3  # hist 2 -> 3 pairs, 1 candidate sees 3


# ---- 8. layer pieces against textbook / library definitions ----------------

def test_linear_matches_numpy():
    rng = np.random.default_rng(300)
    x, w, b = rng.standard_normal((7, 5)), rng.standard_normal((5, 6)), rng.standard_normal(6)
    np.testing.assert_allclose(oracle.linear(x, w, b), x @ w + b, rtol=0, atol=1e-12)
    z = x @ w + b
    np.testing.assert_allclose(oracle.linear(x, w, b, apply_silu=True), z / (1 + np.exp(-z)),
                               rtol=0, atol=1e-12)


def test_norm_gate_matches_torch_layer_norm():
    rng = np.random.default_rng(301)
    o, u = rng.standard_normal((9, 16)), rng.standard_normal((9, 16))
    g, be = rng.standard_normal(16), rng.standard_normal(16)
    ref = torch.nn.functional.layer_norm(torch.tensor(o), (16,), torch.tensor(g), torch.tensor(be),
                                         eps=1e-5).numpy() * u
    np.testing.assert_allclose(oracle.norm_gate(o, u, g, be), ref, rtol=0, atol=1e-12)


def test_layer_matches_composition():
    rng = np.random.default_rng(302)
    H, dqk, dv, D = 2, 3, 2, 5
    c = rand_case(rng, [4, 6, 1], H=H, dqk=dqk, dv=dv, nt=[0, 2, 0])
    T = int(c["seq_offsets"][-1])
    W = H * (2 * dv + 2 * dqk)
    x = rng.standard_normal((T, D))
    w1, b1 = rng.standard_normal((D, W)) * 0.5, rng.standard_normal(W) * 0.1
    w2, b2 = rng.standard_normal((H * dv, D)), rng.standard_normal(D)
    gam, bet = 1 + 0.1 * rng.standard_normal(H * dv), 0.1 * rng.standard_normal(H * dv)
    y = oracle.layer_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], x, w1, b1, w2, b2,
                         gam, bet, c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"],
                         c["inv_n"], H, dqk, dv)
    z = torch.nn.functional.silu(torch.tensor(x) @ torch.tensor(w1) + torch.tensor(b1)).numpy()
    u = z[:, : H * dv]
    vv = z[:, H * dv: 2 * H * dv].reshape(T, H, dv)
    qq = z[:, 2 * H * dv: 2 * H * dv + H * dqk].reshape(T, H, dqk)
    kk = z[:, 2 * H * dv + H * dqk:].reshape(T, H, dqk)
    o = dense_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], qq, kk, vv, c["rab_pos"],
                  c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"]).reshape(T, H * dv)
    g = torch.nn.functional.layer_norm(torch.tensor(o), (H * dv,), torch.tensor(gam),
                                       torch.tensor(bet), eps=1e-5).numpy() * u
    np.testing.assert_allclose(y, g @ w2 + b2, rtol=0, atol=1e-10)
    # output projection over [U | O | G] (3 h d_v wide): each block meets its own rows of W2
    w2c = rng.standard_normal((3 * H * dv, D))
    yc = oracle.layer_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], x, w1, b1, w2c, b2,
                          gam, bet, c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"],
                          c["inv_n"], H, dqk, dv, out_cat=True)
    hv = H * dv
    np.testing.assert_allclose(yc, u @ w2c[:hv] + o @ w2c[hv:2 * hv] + g @ w2c[2 * hv:] + b2, rtol=0, atol=1e-10)


# ---- 8. layer backward: torch float64 autograd and finite differences --------

def _layer_case(seed, lengths=(4, 6, 1), nt=(0, 2, 0), H=2, dqk=3, dv=3, D=5, out_cat=False):
    rng = np.random.default_rng(seed)
    c = rand_case(rng, list(lengths), H=H, dqk=dqk, dv=dv, nt=list(nt))
    T = int(c["seq_offsets"][-1])
    W = H * (2 * dv + 2 * dqk)
    F = (3 if out_cat else 1) * H * dv
    prm = {"x": rng.standard_normal((T, D)), "w1": rng.standard_normal((D, W)) * 0.5,
           "b1": rng.standard_normal(W) * 0.1, "w2": rng.standard_normal((F, D)),
           "b2": rng.standard_normal(D), "ln_gamma": 1 + 0.1 * rng.standard_normal(H * dv),
           "ln_beta": 0.1 * rng.standard_normal(H * dv), "rab_pos": c["rab_pos"], "rab_time": c["rab_time"]}
    dy = rng.standard_normal((T, D))
    return c, prm, dy, (H, dqk, dv)


def _torch_layer_loss(c, prm, dy, dims):
    """sum(Y * dy) of the layer written with torch ops (dense masked attention)."""
    H, dqk, dv = dims
    t = {k: torch.tensor(v, requires_grad=True) for k, v in prm.items()}
    T = prm["x"].shape[0]
    hv, hq = H * dv, H * dqk
    a = torch.nn.functional.silu(t["x"] @ t["w1"] + t["b1"])
    u = a[:, :hv]
    vv = a[:, hv:2 * hv].reshape(T, H, dv)
    qq = a[:, 2 * hv:2 * hv + hq].reshape(T, H, dqk)
    kk = a[:, 2 * hv + hq:].reshape(T, H, dqk)
    off, nt = c["seq_offsets"], c["num_targets"]
    lo, hi = c["pos_lo"], c["pos_hi"]
    outs = []
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        hist = L - n_t
        idx = np.arange(L)
        p = np.where(idx < hist, idx, hist)
        rel = torch.tensor(np.clip(p[:, None] - p[None, :], lo, hi) - lo)
        ts = c["timestamps"][s0:s1]
        nbk = len(prm["rab_time"])
        bkt = torch.tensor([[min(nbk - 1, (int(max(ts[i] - ts[j], 0)) + 1).bit_length() - 1)
                             for j in range(L)] for i in range(L)])
        I, J = idx[:, None], idx[None, :]
        vis = torch.tensor(np.where(I < hist, J <= I, (J < hist) | (J == I)), dtype=torch.float64)
        S = torch.einsum("ihc,jhc->hij", qq[s0:s1], kk[s0:s1]) + (t["rab_pos"][rel] + t["rab_time"][bkt])[None]
        P = torch.nn.functional.silu(S) * c["inv_n"] * vis[None]
        outs.append(torch.einsum("hij,jhc->ihc", P, vv[s0:s1]).reshape(L, hv))
    o = torch.cat(outs)
    g = torch.nn.functional.layer_norm(o, (hv,), t["ln_gamma"], t["ln_beta"], eps=1e-5) * u
    if prm["w2"].shape[0] == 3 * hv:  # output projection over [U | O | G]
        g = torch.cat([u, o, g], dim=1)
    y = g @ t["w2"] + t["b2"]
    (y * torch.tensor(dy)).sum().backward()
    return {k: v.grad.numpy() for k, v in t.items()}


def _olayer_bwd(c, prm, dy, dims):
    H, dqk, dv = dims
    return oracle.layer_bwd(c["seq_offsets"], c["timestamps"], c["num_targets"], prm["x"], prm["w1"],
                            prm["b1"], prm["w2"], prm["ln_gamma"], prm["ln_beta"], prm["rab_pos"],
                            prm["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"], H, dqk, dv, dy,
                            out_cat=prm["w2"].shape[0] == 3 * H * dv)


_LAYER_GRAD_NAMES = {"x": "dx", "w1": "dw1", "b1": "db1", "w2": "dw2", "b2": "db2", "ln_gamma": "d_ln_gamma",
                     "ln_beta": "d_ln_beta", "rab_pos": "d_rab_pos", "rab_time": "d_rab_time"}


@pytest.mark.parametrize("seed,out_cat", [(0, False), (1, False), (2, True), (3, True)])
def test_layer_bwd_matches_torch_autograd(seed, out_cat):
    c, prm, dy, dims = _layer_case(400 + seed, out_cat=out_cat)
    ours = _olayer_bwd(c, prm, dy, dims)
    ref = _torch_layer_loss(c, prm, dy, dims)
    for k, name in _LAYER_GRAD_NAMES.items():
        np.testing.assert_allclose(ours[name], ref[k], rtol=1e-9, atol=1e-10, err_msg=name)


@pytest.mark.parametrize("out_cat", [False, True])
def test_layer_bwd_central_finite_differences(out_cat):
    c, prm, dy, dims = _layer_case(410, lengths=(3, 2), nt=(1, 0), H=1, dqk=2, dv=2, D=3, out_cat=out_cat)
    H, dqk, dv = dims
    ours = _olayer_bwd(c, prm, dy, dims)

    def loss(p):
        y = oracle.layer_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], p["x"], p["w1"], p["b1"],
                             p["w2"], p["b2"], p["ln_gamma"], p["ln_beta"], p["rab_pos"], p["rab_time"],
                             c["pos_lo"], c["pos_hi"], c["inv_n"], H, dqk, dv, out_cat=out_cat)
        return float(np.sum(y * dy))

    h = 1e-6
    rng = np.random.default_rng(411)
    for k, name in _LAYER_GRAD_NAMES.items():
        flat = prm[k].reshape(-1)
        for e in rng.choice(flat.size, size=min(flat.size, 6), replace=False):
            plus, minus = dict(prm), dict(prm)
            fp, fm = flat.copy(), flat.copy()
            fp[e] += h
            fm[e] -= h
            plus[k], minus[k] = fp.reshape(prm[k].shape), fm.reshape(prm[k].shape)
            fd = (loss(plus) - loss(minus)) / (2 * h)
            assert abs(fd - ours[name].reshape(-1)[e]) < 1e-6 * max(1.0, abs(fd)), (name, e, fd)


# ---- 9. semi-local windows ----------------------------------------------------

def _window_mask(L, n_t, local, glob):
    """Independent restatement: causal/candidate rule AND (p_i - p_j < local or j < glob)."""
    hist = L - n_t
    idx = np.arange(L)
    p = np.where(idx < hist, idx, hist)
    I, J = idx[:, None], idx[None, :]
    base = np.where(I < hist, J <= I, (J < hist) | (J == I))
    if local <= 0:
        return base
    return base & (((p[:, None] - p[None, :]) < local) | (J < glob))


def _dense_sl(c, local, glob, dout=None):
    """Dense torch float64 forward (and, with dout, autograd backward) under the windows."""
    off, nt = c["seq_offsets"], c["num_targets"]
    lo, hi = c["pos_lo"], c["pos_hi"]
    t = {k: torch.tensor(c[k], requires_grad=True) for k in ("q", "k", "v", "rab_pos", "rab_time")}
    outs = []
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        hist = L - n_t
        idx = np.arange(L)
        p = np.where(idx < hist, idx, hist)
        rel = torch.tensor(np.clip(p[:, None] - p[None, :], lo, hi) - lo)
        ts = c["timestamps"][s0:s1]
        nbk = len(c["rab_time"])
        bkt = torch.tensor([[min(nbk - 1, (int(max(ts[i] - ts[j], 0)) + 1).bit_length() - 1)
                             for j in range(L)] for i in range(L)])
        vis = torch.tensor(_window_mask(L, n_t, local, glob), dtype=torch.float64)
        S = torch.einsum("ihc,jhc->hij", t["q"][s0:s1], t["k"][s0:s1]) + (t["rab_pos"][rel] + t["rab_time"][bkt])[None]
        P = torch.nn.functional.silu(S) * c["inv_n"] * vis[None]
        outs.append(torch.einsum("hij,jhc->ihc", P, t["v"][s0:s1]))
    o = torch.cat(outs)
    if dout is None:
        return o.detach().numpy()
    (o * torch.tensor(dout)).sum().backward()
    return [t[k].grad.numpy() for k in ("q", "k", "v", "rab_pos", "rab_time")]


def test_visible_sl_exhaustive():
    for L in range(0, 9):
        for n_t in range(0, L + 1):
            for local in range(0, L + 2):
                for glob in range(0, L + 1):
                    m = _window_mask(L, n_t, local, glob)
                    for i in range(L):
                        for j in range(L):
                            assert oracle.visible_sl(i, j, L, n_t, local, glob) == bool(m[i, j])


@pytest.mark.parametrize("local,glob", [(3, 0), (2, 2), (5, 1), (1, 3)])
def test_semi_local_matches_dense(local, glob):
    rng = np.random.default_rng(500 + 7 * local + glob)
    c = rand_case(rng, [7, 1, 0, 9], nt=[2, 0, 0, 3])
    args = (c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"], c["rab_pos"],
            c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])
    o = oracle.attn_fwd(*args, local_window=local, global_window=glob)
    np.testing.assert_allclose(o, _dense_sl(c, local, glob), rtol=0, atol=1e-12)
    dout = rng.standard_normal(c["v"].shape)
    ours = oracle.attn_bwd(*args, dout, local_window=local, global_window=glob)
    for a, b in zip(ours, _dense_sl(c, local, glob, dout)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_semi_local_limits():
    rng = np.random.default_rng(520)
    c = rand_case(rng, [6, 4], nt=[1, 0])
    args = (c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"], c["rab_pos"],
            c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])
    full = oracle.attn_fwd(*args)
    # a local window covering every distance, or a global window covering every key, is the full mask
    np.testing.assert_array_equal(oracle.attn_fwd(*args, local_window=100, global_window=0), full)
    np.testing.assert_array_equal(oracle.attn_fwd(*args, local_window=1, global_window=100), full)
    # local 1, no global keys: only the diagonal, O_i = SiLU(s_ii) / N v_i
    o = oracle.attn_fwd(*args, local_window=1, global_window=0)
    off, nt = c["seq_offsets"], c["num_targets"]
    for b in range(2):
        s0, L = int(off[b]), int(off[b + 1] - off[b])
        for i in range(L):
            idx = int(np.clip(0, c["pos_lo"], c["pos_hi"]) - c["pos_lo"])
            s = np.einsum("hc,hc->h", c["q"][s0 + i], c["k"][s0 + i]) + c["rab_pos"][idx] + c["rab_time"][0]
            expect = (s / (1 + np.exp(-s)) * c["inv_n"])[:, None] * c["v"][s0 + i]
            np.testing.assert_allclose(o[s0 + i], expect, rtol=0, atol=1e-12)
    # the call leaves no windows behind
    np.testing.assert_array_equal(oracle.attn_fwd(*args), full)


def test_semi_local_pair_counter_by_brute_force():
    for L in range(0, 12):
        for n_t in range(0, L + 1):
            for w in range(0, L + 2):
                for g in range(0, L + 1):
                    brute = sum(oracle.visible_sl(i, j, L, n_t, w, g) for i in range(L) for j in range(L))
                    assert flops.attn_pairs_per_seq(L, n_t, w, g) == brute, (L, n_t, w, g)


# ---- attention truncation (segment gather) -----------------------------------

def test_truncate_hand_worked():
    g = _parse_golden("truncate_hand.txt")
    off = np.asarray(g["seq_offsets"], np.int64)
    nt = np.asarray(g["num_targets"], np.int32)
    rows = np.arange(11, dtype=np.float64)
    for keep in (0, 1, 2):
        new_off, kept = oracle.jagged_truncate(off, nt, keep, rows)
        np.testing.assert_array_equal(new_off, g[f"keep{keep}_offsets"])
        np.testing.assert_array_equal(kept, g[f"keep{keep}_rows"])


def test_truncate_limits():
    rng = np.random.default_rng(700)
    lengths = np.array([0, 1, 5, 9, 3])
    nt = np.array([0, 1, 2, 0, 3], np.int32)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    rows = rng.standard_normal((int(off[-1]), 3))
    # a segment at least as long as every history keeps everything
    new_off, kept = oracle.jagged_truncate(off, nt, 9, rows)
    np.testing.assert_array_equal(new_off, off)
    np.testing.assert_array_equal(kept, rows)
    # each sequence keeps min(hist, keep) + n_t tokens, and its last ones
    for keep in range(0, 10):
        new_off, kept = oracle.jagged_truncate(off, nt, keep, rows)
        np.testing.assert_array_equal(np.diff(new_off), np.minimum(lengths - nt, keep) + nt)
        for b in range(len(lengths)):
            n = int(new_off[b + 1] - new_off[b])
            np.testing.assert_array_equal(kept[new_off[b]:new_off[b + 1]], rows[off[b + 1] - n:off[b + 1]])
    # no candidate information: every token is history
    new_off, _ = oracle.jagged_truncate(off, None, 2, rows)
    np.testing.assert_array_equal(np.diff(new_off), np.minimum(lengths, 2))
    # empty batch
    new_off, kept = oracle.jagged_truncate(np.zeros(1, np.int64), None, 4, rows[:0])
    assert new_off.tolist() == [0] and len(kept) == 0


def test_truncated_candidates_see_a_local_window():
    # A candidate of the truncated sequence attends to the `keep` most recent
    # history tokens and itself; relative positions and time gaps are unchanged
    # by the cut, so its output equals the full sequence's with a local window
    # of keep + 1 positions and no global window.
    rng = np.random.default_rng(710)
    c = rand_case(rng, [9, 4, 7], nt=[2, 1, 3])
    for keep in (0, 2, 3, 6):
        off, nt = c["seq_offsets"], c["num_targets"]
        new_off, ts = oracle.jagged_truncate(off, nt, keep, c["timestamps"])
        q, k, v = (oracle.jagged_truncate(off, nt, keep, c[n])[1] for n in ("q", "k", "v"))
        cut = oracle.attn_fwd(new_off, ts, nt, q, k, v, c["rab_pos"], c["rab_time"], c["pos_lo"],
                              c["pos_hi"], c["inv_n"])
        win = oracle.attn_fwd(off, c["timestamps"], nt, c["q"], c["k"], c["v"], c["rab_pos"],
                              c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"], local_window=keep + 1,
                              global_window=0)
        for b in range(3):
            n_t = int(nt[b])
            np.testing.assert_allclose(cut[new_off[b + 1] - n_t:new_off[b + 1]], win[off[b + 1] - n_t:off[b + 1]],
                                       rtol=0, atol=1e-13)


def test_windowed_layer_is_the_composition_with_windowed_attention():
    # the layer's attention takes the same windows as the attention alone (pinned above)
    rng = np.random.default_rng(730)
    H, dqk, dv, D = 2, 3, 2, 5
    c = rand_case(rng, [9, 4, 12], H=H, dqk=dqk, dv=dv, nt=[2, 0, 3])
    T = int(c["seq_offsets"][-1])
    W = H * (2 * dv + 2 * dqk)
    x = rng.standard_normal((T, D))
    w1, b1 = rng.standard_normal((D, W)) * 0.5, rng.standard_normal(W) * 0.1
    w2, b2 = rng.standard_normal((H * dv, D)), rng.standard_normal(D)
    gam, bet = 1 + 0.1 * rng.standard_normal(H * dv), 0.1 * rng.standard_normal(H * dv)
    args = (c["seq_offsets"], c["timestamps"], c["num_targets"])
    tables = (c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])
    y = oracle.layer_fwd(*args, x, w1, b1, w2, b2, gam, bet, *tables, H, dqk, dv, local_window=3, global_window=2)
    a = oracle.linear(x, w1, b1, apply_silu=True)
    hv, hq = H * dv, H * dqk
    o = oracle.attn_fwd(*args, a[:, 2 * hv:2 * hv + hq].reshape(T, H, dqk), a[:, 2 * hv + hq:].reshape(T, H, dqk),
                        a[:, hv:2 * hv].reshape(T, H, dv), *tables, local_window=3, global_window=2)
    g = oracle.norm_gate(o.reshape(T, hv), a[:, :hv], gam, bet)
    np.testing.assert_allclose(y, oracle.linear(g, w2, b2), rtol=0, atol=1e-12)
    # and differs from the full-mask layer
    assert np.abs(y - oracle.layer_fwd(*args, x, w1, b1, w2, b2, gam, bet, *tables, H, dqk, dv)).max() > 1e-6


# ---- visible pairs per bias entry --------------------------------------------

def _counts(lengths, ts, nts=None, lo=0, hi=10**6, nb=64, local=0, glob=0):
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return oracle.bias_pair_counts(off, np.asarray(ts, dtype=np.int64), nts, lo, hi, nb, local, glob)


def test_bias_pair_counts_causal_unit_gaps_closed_form():
    # one causal sequence with stamps t_j = j: distance k = i - j occurs L - k times,
    # and bucket b holds the distances 2^b - 1 .. 2^(b+1) - 2 (the last bucket the rest)
    L, nb = 300, 6
    pc, tc = _counts([L], np.arange(L), lo=0, hi=L - 1, nb=nb)
    assert list(pc) == [L - k for k in range(L)]
    exp = []
    for b in range(nb):
        lo_d = 2 ** b - 1
        hi_d = 2 ** (b + 1) - 2 if b < nb - 1 else L - 1
        exp.append(sum(L - d for d in range(lo_d, min(hi_d, L - 1) + 1)))
    assert list(tc) == exp
    assert tc.sum() == pc.sum() == L * (L + 1) // 2


def test_bias_pair_counts_clamps_closed_form():
    L, lo, hi = 120, 2, 40
    pc, _ = _counts([L], np.zeros(L), lo=lo, hi=hi, nb=4)
    assert pc[0] == sum(L - d for d in range(0, lo + 1))          # distances 0..2 clamp to 2
    assert pc[-1] == (L - hi) * (L - hi + 1) // 2                 # distances >= 40 clamp to 40
    assert list(pc[1:-1]) == [L - d for d in range(lo + 1, hi)]


def test_bias_pair_counts_candidates_closed_form():
    # 43 history tokens + 7 candidates at position 43 with the last history stamp:
    # history pairs as before, each candidate adds one pair at distances 1..43 and its own at 0
    hist, nt = 43, 7
    L = hist + nt
    ts = np.concatenate([np.arange(hist) * 5, np.full(nt, (hist - 1) * 5)])
    pc, tc = _counts([L], ts, nts=np.array([nt], dtype=np.int32), lo=0, hi=100, nb=40)
    exp = np.zeros(101, dtype=np.int64)
    for k in range(hist):
        exp[k] += hist - k
    exp[1:hist + 1] += nt
    exp[0] += nt
    assert np.array_equal(pc, exp)
    assert tc.sum() == hist * (hist + 1) // 2 + nt * (hist + 1)
    # a candidate and its own pair: dt = 0 -> bucket 0, as for every diagonal pair
    assert tc[0] >= hist + nt


def test_bias_pair_counts_local_window_closed_form():
    # causal, local window 10, first 3 keys global: distance k < 10 keeps all L - k pairs,
    # a larger distance only the pairs whose key is global
    L, w, g = 100, 10, 3
    pc, _ = _counts([L], np.arange(L), lo=0, hi=L - 1, nb=8, local=w, glob=g)
    exp = [L - k if k < w else min(g, L - k) for k in range(L)]
    assert list(pc) == exp


def test_bias_pair_counts_by_brute_force():
    # random tiny batch with candidates, windows, unsorted stamps and an empty sequence,
    # against loops over the scalar visibility and index functions
    rng = np.random.default_rng(3)
    lengths, nts = [9, 0, 14, 5], np.array([2, 0, 4, 0], dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    ts = rng.integers(0, 3000, size=off[-1]).astype(np.int64)
    lo, hi, nb, w, g = -2, 6, 7, 4, 2
    pc, tc = oracle.bias_pair_counts(off, ts, nts, lo, hi, nb, w, g)
    epc, etc = np.zeros_like(pc), np.zeros_like(tc)
    for b, L in enumerate(lengths):
        n = int(nts[b])
        hist = L - n
        for i in range(L):
            for j in range(L):
                if not oracle.visible_sl(i, j, L, n, w, g):
                    continue
                epc[oracle.pos_index(min(i, hist), min(j, hist), lo, hi)] += 1
                etc[oracle.time_bucket(ts[off[b] + i], ts[off[b] + j], nb)] += 1
    assert np.array_equal(pc, epc) and np.array_equal(tc, etc)


def test_bias_pair_counts_are_the_uniform_score_gradient():
    # q = k = 0 and zero tables give s = 0 on every visible pair; with v = dout = 1 every
    # pair's dS is d_v SiLU'(0) / N = d_v / (2N), so the backward's table gradients are
    # H d_v / (2N) times the pair counts (the backward is pinned by finite differences)
    rng = np.random.default_rng(8)
    lengths, nts = [12, 7, 0, 20], np.array([3, 0, 0, 5], dtype=np.int32)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T, H, d, lo, hi, nb, inv_n = int(off[-1]), 2, 4, -3, 9, 6, 1 / 16
    ts = np.cumsum(rng.integers(0, 40, size=T)).astype(np.int64)
    z = np.zeros((T, H, d))
    one = np.ones((T, H, d))
    for w, g in [(0, 0), (5, 2)]:
        _, _, _, drp, drt = oracle.attn_bwd(off, ts, nts, z, z, one, np.zeros(hi - lo + 1), np.zeros(nb),
                                            lo, hi, inv_n, one, local_window=w, global_window=g)
        pc, tc = oracle.bias_pair_counts(off, ts, nts, lo, hi, nb, w, g)
        assert np.array_equal(drp, pc * (H * d * 0.5 * inv_n))
        assert np.array_equal(drt, tc * (H * d * 0.5 * inv_n))


# ---- readings selected per call: candidates at their own index, per-head tables ----

def dense_fwd_readings(c, own=False):
    """Dense forward (numpy) with candidate positions at their own index when `own`
    and per-head tables when rab_pos is [H, entries]."""
    off, ts, nt = c["seq_offsets"], c["timestamps"], c["num_targets"]
    q, k, v, lo, hi = c["q"], c["k"], c["v"], c["pos_lo"], c["pos_hi"]
    T, H, dv = v.shape
    rp, rt = np.asarray(c["rab_pos"]), np.asarray(c["rab_time"])
    if rp.ndim == 1:
        rp, rt = np.stack([rp] * H), np.stack([rt] * H)
    nb = rt.shape[1]
    out = np.zeros((T, H, dv))
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        hist = L - n_t
        idx = np.arange(L)
        p = idx if own else np.where(idx < hist, idx, hist)
        rel = np.clip(p[:, None] - p[None, :], lo, hi) - lo
        t = ts[s0:s1]
        dt = np.maximum(t[:, None].astype(object) - t[None, :].astype(object), 0)
        bkt = np.vectorize(lambda x: min(nb - 1, (int(x) + 1).bit_length() - 1), otypes=[np.int64])(dt)
        I, J = idx[:, None], idx[None, :]
        vis = np.where(I < hist, J <= I, (J < hist) | (J == I))
        S = np.einsum("ihc,jhc->hij", q[s0:s1], k[s0:s1]) + np.stack([rp[h][rel] + rt[h][bkt] for h in range(H)])
        P = S / (1.0 + np.exp(-S)) * c["inv_n"] * vis[None]
        out[s0:s1] = np.einsum("hij,jhc->ihc", P, v[s0:s1])
    return out


def _per_head_case(rng, lengths, nt, H=3):
    c = rand_case(rng, lengths, H=H, nt=nt)
    c["rab_pos"] = rng.standard_normal((H, c["pos_hi"] - c["pos_lo"] + 1)) * 0.3
    c["rab_time"] = rng.standard_normal((H, 5)) * 0.3
    return c


@pytest.mark.parametrize("seed", range(3))
def test_own_index_candidates_match_dense(seed):
    rng = np.random.default_rng(300 + seed)
    lengths = [9, 6, 1, 11]
    nt = [3, 6, 1, 4]
    c = rand_case(rng, lengths, nt=nt, lo=-2, hi=12)
    got = oracle.attn_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                          c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"], cand_own_index=True)
    np.testing.assert_allclose(got, dense_fwd_readings(c, own=True), rtol=0, atol=1e-12)
    # the two readings differ only through the candidates' positions
    shared = ofwd(c)
    no_cand = dict(c, num_targets=None)
    np.testing.assert_array_equal(oracle.attn_fwd(no_cand["seq_offsets"], no_cand["timestamps"], None, c["q"], c["k"],
                                                  c["v"], c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"],
                                                  c["inv_n"], cand_own_index=True), ofwd(no_cand))
    assert np.abs(dense_fwd_readings(c, own=True) - shared).max() > 1e-6


@pytest.mark.parametrize("seed", range(3))
def test_per_head_tables_match_dense(seed):
    rng = np.random.default_rng(320 + seed)
    c = _per_head_case(rng, [7, 0, 10, 3], [2, 0, 0, 1])
    got = oracle.attn_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                          c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])
    np.testing.assert_allclose(got, dense_fwd_readings(c), rtol=0, atol=1e-12)


def test_per_head_tables_identical_heads_are_the_shared_tables():
    rng = np.random.default_rng(340)
    c = rand_case(rng, [8, 5, 12], H=3, nt=[0, 2, 4])
    H = 3
    per = dict(c, rab_pos=np.stack([c["rab_pos"]] * H), rab_time=np.stack([c["rab_time"]] * H))
    args = lambda d: (d["seq_offsets"], d["timestamps"], d["num_targets"], d["q"], d["k"], d["v"], d["rab_pos"],
                      d["rab_time"], d["pos_lo"], d["pos_hi"], d["inv_n"])
    np.testing.assert_array_equal(oracle.attn_fwd(*args(per)), oracle.attn_fwd(*args(c)))
    dout = rng.standard_normal(c["v"].shape)
    g_shared = oracle.attn_bwd(*args(c), dout)
    g_per = oracle.attn_bwd(*args(per), dout)
    for a, b in zip(g_per[:3], g_shared[:3]):
        np.testing.assert_array_equal(a, b)
    assert g_per[3].shape == (H, c["rab_pos"].size) and g_per[4].shape == (H, c["rab_time"].size)
    np.testing.assert_allclose(g_per[3].sum(axis=0), g_shared[3], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g_per[4].sum(axis=0), g_shared[4], rtol=0, atol=1e-12)


def test_per_head_tables_heads_are_independent():
    # head h of a per-head problem is the one-head problem with head h's inputs and tables
    rng = np.random.default_rng(350)
    c = _per_head_case(rng, [9, 4], [2, 0])
    dout = rng.standard_normal(c["v"].shape)
    full = oracle.attn_bwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                           c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"], dout)
    fo = oracle.attn_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                         c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"])
    for h in range(3):
        sl = slice(h, h + 1)
        one = oracle.attn_bwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"][:, sl], c["k"][:, sl],
                              c["v"][:, sl], c["rab_pos"][h], c["rab_time"][h], c["pos_lo"], c["pos_hi"], c["inv_n"],
                              dout[:, sl])
        of = oracle.attn_fwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"][:, sl], c["k"][:, sl],
                             c["v"][:, sl], c["rab_pos"][h], c["rab_time"][h], c["pos_lo"], c["pos_hi"], c["inv_n"])
        np.testing.assert_array_equal(fo[:, sl], of)
        for a, b in zip(full[:3], one[:3]):
            np.testing.assert_array_equal(a[:, sl], b)
        np.testing.assert_array_equal(full[3][h], one[3])
        np.testing.assert_array_equal(full[4][h], one[4])


def _torch_dense_loss_readings(c, dout, own):
    off, nt = c["seq_offsets"], c["num_targets"]
    q = torch.tensor(c["q"], requires_grad=True)
    k = torch.tensor(c["k"], requires_grad=True)
    v = torch.tensor(c["v"], requires_grad=True)
    rp = torch.tensor(np.asarray(c["rab_pos"]), requires_grad=True)
    rt = torch.tensor(np.asarray(c["rab_time"]), requires_grad=True)
    H = c["q"].shape[1]
    lo, hi = c["pos_lo"], c["pos_hi"]
    loss = 0.0
    for b in range(len(off) - 1):
        s0, s1 = int(off[b]), int(off[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        n_t = 0 if nt is None else int(nt[b])
        hist = L - n_t
        idx = np.arange(L)
        p = idx if own else np.where(idx < hist, idx, hist)
        rel = torch.tensor(np.clip(p[:, None] - p[None, :], lo, hi) - lo)
        ts = c["timestamps"][s0:s1]
        nb = rt.shape[-1]
        bkt = torch.tensor([[min(nb - 1, (int(max(ts[i] - ts[j], 0)) + 1).bit_length() - 1)
                             for j in range(L)] for i in range(L)])
        I, J = idx[:, None], idx[None, :]
        vis = torch.tensor(np.where(I < hist, J <= I, (J < hist) | (J == I)), dtype=torch.float64)
        if rp.dim() == 2:
            bias = torch.stack([rp[h][rel] + rt[h][bkt] for h in range(H)])
        else:
            bias = (rp[rel] + rt[bkt])[None]
        S = torch.einsum("ihc,jhc->hij", q[s0:s1], k[s0:s1]) + bias
        P = torch.nn.functional.silu(S) * c["inv_n"] * vis[None]
        O = torch.einsum("hij,jhc->ihc", P, v[s0:s1])
        loss = loss + (O * torch.tensor(dout[s0:s1])).sum()
    loss.backward()
    return [x.grad.numpy() for x in (q, k, v, rp, rt)]


@pytest.mark.parametrize("own,per_head", [(True, False), (False, True), (True, True)])
def test_readings_bwd_match_torch_autograd(own, per_head):
    rng = np.random.default_rng(360 + 2 * own + per_head)
    lengths, nt = [7, 3, 9], [2, 3, 4]
    c = _per_head_case(rng, lengths, nt) if per_head else rand_case(rng, lengths, H=3, nt=nt)
    dout = rng.standard_normal(c["v"].shape)
    ours = oracle.attn_bwd(c["seq_offsets"], c["timestamps"], c["num_targets"], c["q"], c["k"], c["v"],
                           c["rab_pos"], c["rab_time"], c["pos_lo"], c["pos_hi"], c["inv_n"], dout,
                           cand_own_index=own)
    ref = _torch_dense_loss_readings(c, dout, own)
    for a, b in zip(ours, ref):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_bias_pair_counts_own_index_candidates_closed_form():
    # candidate i (own position i) sees every history key j at distance i - j and itself at 0
    hist, nt = 20, 5
    L = hist + nt
    pc, tc = _counts([L], np.arange(L), nts=np.array([nt], dtype=np.int32), lo=0, hi=100, nb=10)
    own = oracle.bias_pair_counts(np.array([0, L]), np.arange(L), np.array([nt], dtype=np.int32), 0, 100, 10,
                                  cand_own_index=True)[0]
    exp = np.zeros(101, dtype=np.int64)
    for k in range(hist):
        exp[k] += hist - k
    for i in range(hist, L):
        for j in range(hist):
            exp[i - j] += 1
        exp[0] += 1
    np.testing.assert_array_equal(own, exp)
    assert own.sum() == pc.sum()
