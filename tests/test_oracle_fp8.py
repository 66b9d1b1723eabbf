"""Pins of the oracle's FP8 (E4M3) codec, quantisers and projections.

The codec is pinned by the format's closed forms (largest finite 448, smallest
normal 2^-6, smallest subnormal 2^-9), hand-worked ties, the round trip of
every finite code and torch's own float8_e4m3fn conversion (the library
routine) on in-range values; the quantisers by their defining properties; the
GEMM by a numpy matmul of the decoded operands."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8


def test_decode_closed_forms():
    d = fp8.e4m3_decode
    assert d(0x38) == 1.0 and d(0xB8) == -1.0
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0
    assert d(0x08) == 2.0 ** -6            # smallest normal
    assert d(0x01) == 2.0 ** -9            # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9        # largest subnormal
    assert d(0x3F) == 1.875 and d(0x40) == 2.0
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))
    assert d(0x00) == 0.0 and d(0x80) == 0.0


def test_encode_hand_worked_ties_and_saturation():
    e = lambda v: int(fp8.e4m3_encode(np.float32(v)))
    assert e(1.0625) == 0x38       # halfway 1 / 1.125: even code 0x38
    assert e(1.1875) == 0x3A       # halfway 1.125 / 1.25: even code 0x3A
    assert e(1.07) == 0x39         # above halfway
    assert e(2.0 ** -10) == 0x00   # halfway 0 / 2^-9: even code 0
    assert e(3 * 2.0 ** -10) == 0x02
    assert e(460.0) == 0x7E        # below the midpoint to 480: 448
    assert e(1e6) == 0x7E and e(-1e6) == 0xFE  # saturated
    assert e(-2.0 ** -11) == 0x80  # rounds to zero, keeps the sign


def test_round_trip_of_every_finite_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    back = fp8.e4m3_encode(fp8.e4m3_decode(codes).astype(np.float32))
    np.testing.assert_array_equal(back, codes)


def test_encode_matches_torch_float8_in_range():
    rng = np.random.default_rng(900)
    mant = rng.uniform(-1, 1, 200000)
    expo = rng.integers(-14, 9, 200000)
    v = (mant * np.exp2(expo)).astype(np.float32)
    v = v[np.abs(v) < 464.0]  # torch does not saturate; below 464 both round the same way
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fp8.e4m3_encode(v), ref)


def test_quantize_rows_properties():
    rng = np.random.default_rng(901)
    x = (rng.standard_normal((50, 96)) * np.exp2(rng.integers(-8, 8, (50, 1)))).astype(np.float32)
    x[3] = 0.0
    codes, scale = fp8.quantize_rows(x)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    mag = codes & 0x7F
    # every non-zero row reaches the largest code at its amax, none exceeds it
    for r in range(50):
        if r == 3:
            assert scale[r] == 1.0 and not mag[r].any()
            continue
        assert mag[r].max() == 0x7E and mag[r, np.argmax(np.abs(x[r]))] == 0x7E
    deq = fp8.dequantize(codes, scale)
    # relative error within half a unit of the 3-bit mantissa, plus the subnormal step
    bound = 2.0 ** -4 * np.abs(x) + scale[:, None].astype(np.float64) * 2.0 ** -10
    assert np.all(np.abs(deq - x) <= bound * (1 + 1e-6))
    np.testing.assert_array_equal(np.signbit(deq[x != 0]), np.signbit(x[x != 0]))


def test_quantize_weight_is_per_output_column():
    rng = np.random.default_rng(902)
    w = rng.standard_normal((64, 40)).astype(np.float32)
    codes, scale = fp8.quantize_weight(w)
    assert codes.shape == (40, 64) and scale.shape == (40,)
    np.testing.assert_allclose(scale, np.abs(w).max(axis=0) / 448.0, rtol=1e-7)


def test_gemm_matches_numpy_on_decoded_operands():
    rng = np.random.default_rng(903)
    x = rng.standard_normal((33, 64)).astype(np.float32)
    w = rng.standard_normal((64, 48)).astype(np.float32)
    b = rng.standard_normal(48)
    xq, sx = fp8.quantize_rows(x)
    wq, sw = fp8.quantize_weight(w)
    ref = (fp8.e4m3_decode(xq) * sx[:, None]) @ (fp8.e4m3_decode(wq) * sw[:, None]).T + b
    np.testing.assert_allclose(fp8.gemm(xq, sx, wq, sw, b), ref, rtol=1e-12, atol=1e-12)
    z = ref
    np.testing.assert_allclose(fp8.gemm(xq, sx, wq, sw, b, apply_silu=True), z / (1 + np.exp(-z)),
                               rtol=1e-12, atol=1e-12)


def test_fp8_layer_is_close_to_the_bf16_layer():
    rng = np.random.default_rng(904)
    H, d, D = 2, 8, 32
    lengths = [20, 7, 1]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    ts = np.concatenate([np.cumsum(rng.integers(0, 300, L)) for L in lengths]).astype(np.int64)
    W = H * 4 * d
    x = rng.standard_normal((T, D)).astype(np.float32)
    w1 = (rng.standard_normal((D, W)) * 0.2).astype(np.float32)
    w2 = (rng.standard_normal((H * d, D)) * 0.2).astype(np.float32)
    b1, b2 = rng.standard_normal(W) * 0.1, rng.standard_normal(D) * 0.1
    g, be = 1 + 0.1 * rng.standard_normal(H * d), 0.1 * rng.standard_normal(H * d)
    rp, rt = rng.standard_normal(41) * 0.1, rng.standard_normal(8) * 0.1
    args = (off, ts, None)
    ref = oracle.layer_fwd(*args, x, w1, b1, w2, b2, g, be, rp, rt, -20, 20, 0.05, H, d, d)
    w1q, s1 = fp8.quantize_weight(w1)
    w2q, s2 = fp8.quantize_weight(w2)
    y = fp8.layer_fwd(*args, x, w1q, s1, b1, w2q, s2, b2, g, be, rp, rt, -20, 20, 0.05, H, d, d)
    # 3-bit mantissas: a few percent of the output's range, not more
    err = np.abs(y - ref).max() / np.abs(ref).max()
    assert 1e-4 < err < 0.1, err


def test_fp8_scores_are_exact_when_q_and_k_are_representable():
    # rows whose values are E4M3 codes times a power of two, with the row's largest
    # magnitude at 448 times that power: the quantisation is exact, so the FP8-score
    # attention equals the plain one
    rng = np.random.default_rng(905)
    lengths = [7, 1, 12]
    T, H, d = sum(lengths), 2, 8
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    ts = np.concatenate([np.cumsum(rng.integers(0, 50, L)) for L in lengths]).astype(np.int64)
    finite = np.array([c for c in range(256) if c & 0x7F != 0x7F and c & 0x7F <= 0x7E], np.uint8)

    def exact(shape):
        codes = rng.choice(finite, size=shape)
        codes[..., 0] = 0x7E  # the row's amax maps to 448 exactly
        pw = np.exp2(rng.integers(-12, -6, shape[:-1]))[..., None]
        return fp8.e4m3_decode(codes) * pw

    q, k = exact((T, H, d)), exact((T, H, d))
    v = rng.standard_normal((T, H, d))
    rp, rt = rng.standard_normal(21) * 0.1, rng.standard_normal(6) * 0.1
    args = (off, ts, None)
    ref = oracle.attn_fwd(*args, q, k, v, rp, rt, -10, 10, 0.1)
    np.testing.assert_allclose(fp8.attn_fwd_qk(*args, q, k, v, rp, rt, -10, 10, 0.1), ref, rtol=0, atol=1e-12)
    # general values: within the 3-bit mantissa's error of the plain attention
    q2, k2 = rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d))
    a = fp8.attn_fwd_qk(*args, q2, k2, v, rp, rt, -10, 10, 0.1)
    b = oracle.attn_fwd(*args, q2, k2, v, rp, rt, -10, 10, 0.1)
    err = np.abs(a - b).max() / np.abs(b).max()
    assert 1e-4 < err < 0.1, err
