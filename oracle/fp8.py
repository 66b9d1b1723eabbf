"""FP8 (E4M3) projections and scores for the oracle.  TEST INFRASTRUCTURE ONLY, like the
rest of `oracle/`: only the tests, the smoke check and the bench's CPU leg use it.

The ULTRA-HSTU review in the pages (its mixed-precision item) keeps most of the
layer in bf16 and runs the matrix multiplications in FP8.  The pages fix neither
the FP8 format nor the scaling; the readings taken here are:
  * format E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest
    finite 448, no infinities), values rounded to nearest, ties to even, and
    saturated to +-448;
  * activations scaled per row (token), weights per output column, each so
    that its largest magnitude maps to 448: with amax the row's (column's)
    largest |value| in float32, inv = 448 / amax and scale = amax / 448 (both
    float32, correctly rounded), code = E4M3(float32(x * inv)), and the value
    a code stands for is decode(code) * scale; an all-zero row has scale 1;
  * the product of two quantised operands is exact and accumulated in float64
    here, then scaled: y[m, n] = sum_k dec(xq[m, k]) dec(wq[n, k]) sx[m] sw[n].
In the FP8 layer only the projections f1 and f2 are quantised; the attention
and the gate stay as in the bf16 layer.  The FP8-score attention (attn_fwd_qk)
quantises q and k per (token, head) row the same way and keeps P V in bf16:
the pages name the product QK^T and AV together, and the reading taken keeps P
and V out of FP8, since a row's P has no scale known before all its key tiles.
"""

from __future__ import annotations

import numpy as np

from . import attn_fwd, linear, norm_gate

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (float64; NaN for the two NaN codes)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return sign * v


# the 127 non-negative finite codes, in increasing order of value
_POS_CODES = np.arange(0, 0x7F, dtype=np.int64)
_POS_VALUES = e4m3_decode(_POS_CODES)


def e4m3_encode(v) -> np.ndarray:
    """Nearest E4M3 code of each float32 value, ties to the even code, magnitudes
    above 448 saturated to 448; the sign bit follows the sign of v (a negative
    value that rounds to zero gives 0x80)."""
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(_POS_VALUES, a, side="left"), 0, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - _POS_VALUES[lo], _POS_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    neg = np.signbit(v)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def quantize_rows(x):
    """Per-row E4M3 quantisation of x [R, K] (float32 arithmetic): (codes uint8
    [R, K], scales float32 [R])."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    amax = amax.astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    scale = np.where(amax > 0, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    codes = e4m3_encode((x * inv[:, None]).astype(np.float32))
    return codes, scale


def quantize_weight(w):
    """Per-output-column quantisation of a weight w [K, N]: (codes uint8 [N, K],
    the transposed layout, scales float32 [N])."""
    if hasattr(w, "detach"):
        w = w.detach().cpu().float().numpy()
    return quantize_rows(np.asarray(w, dtype=np.float32).T)


def dequantize(codes, scales):
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]


def gemm(xq, sx, wq, sw, bias=None, apply_silu=False):
    """y = (dec(xq) sx) (dec(wq) sw)^T + bias, optionally SiLU (float64)."""
    return linear(dequantize(xq, sx), dequantize(wq, sw).T, bias, apply_silu)


def layer_fwd(seq_offsets, timestamps, num_targets, x, w1q, s1, b1, w2q, s2, b2, ln_gamma, ln_beta, rab_pos,
              rab_time, pos_lo, pos_hi, inv_n, num_heads, d_qk, d_v, ln_eps=1e-5, want_intermediates=False,
              g_round=None):
    """The transduction layer with FP8 projections: X and G quantised per row,
    W1 and W2 given quantised per output column ([N, K] codes and [N] scales).
    The bf16 layer rounds G to bf16 before quantising it; `g_round` (a function
    on a float64 array) applies that rounding here when given."""
    hv, hq = num_heads * d_v, num_heads * d_qk
    xq, sx = quantize_rows(x)
    a = gemm(xq, sx, w1q, s1, b1, apply_silu=True)
    T = a.shape[0]
    u = a[:, :hv]
    v = a[:, hv:2 * hv].reshape(T, num_heads, d_v)
    q = a[:, 2 * hv:2 * hv + hq].reshape(T, num_heads, d_qk)
    k = a[:, 2 * hv + hq:].reshape(T, num_heads, d_qk)
    o = attn_fwd(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi,
                 inv_n).reshape(T, hv)
    g = norm_gate(o, u, ln_gamma, ln_beta, ln_eps)
    if g_round is not None:
        g = g_round(g)
    gq, sg = quantize_rows(g)
    y = gemm(gq, sg, w2q, s2, b2)
    if want_intermediates:
        return y, a, o
    return y


def quantize_heads(x):
    """Per-(token, head) row E4M3 quantisation of q or k [T, H, d]: (codes uint8
    [T, H, d], scales float32 [T, H])."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    x = np.asarray(x, dtype=np.float32)
    T, H, d = x.shape
    codes, scales = quantize_rows(x.reshape(T * H, d))
    return codes.reshape(T, H, d), scales.reshape(T, H)


def attn_fwd_qk(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n,
                **windows):
    """Attention forward with the score product in FP8: q and k quantised per
    (token, head) row, s = dec(q) . dec(k) exactly, the rest (bias, SiLU, P V
    with bf16-valued P and V in the kernels) as in the bf16 attention."""
    qq, sq = quantize_heads(q)
    kq, sk = quantize_heads(k)
    qd = e4m3_decode(qq) * sq[..., None].astype(np.float64)
    kd = e4m3_decode(kq) * sk[..., None].astype(np.float64)
    return attn_fwd(seq_offsets, timestamps, num_targets, qd, kd, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n,
                    **windows)
