"""Algorithmic FLOP and byte accounting for the HSTU hot path.

Follows "DLRMv4 Brings Sequence-Based Recommendation Training to MLPerf",
section "Computation Cost Analysis" (Tables 6 and 7): the attention forward
is two GEMM-shaped contractions (Q K^T and P V), the backward roughly five,
and only the visible (lower-triangle) pairs are counted.  Bias gathers, SiLU
and the mask are not counted.  Weight GEMMs cost 2*m*n*k per pass.
"""

from __future__ import annotations

import numpy as np


def attn_pairs_per_seq(L: int, n_t: int = 0, local_window: int = 0, global_window: int = 0) -> int:
    """Visible (query, key) pairs of one sequence: history rows see j <= i,
    each candidate row sees the whole history and itself.  With local_window
    w > 0 (semi-local attention) a pair also needs p_i - p_j < w or j < g, the
    global window: history row i keeps min(i + 1, w) local keys plus the global
    keys before them, max(0, min(g, i + 1 - w)); a candidate (position hist)
    keeps min(hist, w - 1) local history keys, the global ones before them,
    and itself."""
    L, n_t, w, g = int(L), int(n_t), int(local_window), int(global_window)
    hist = L - n_t
    if w <= 0:
        return hist * (hist + 1) // 2 + n_t * (hist + 1)
    i = np.arange(hist, dtype=np.int64)
    rows = np.minimum(i + 1, w) + np.maximum(0, np.minimum(g, i + 1 - w))
    cand = min(hist, w - 1) + max(0, min(g, hist - w + 1)) + 1
    return int(rows.sum()) + n_t * cand


def attn_pairs(lengths, num_targets=None, local_window: int = 0, global_window: int = 0) -> int:
    lengths = np.asarray(lengths, dtype=np.int64)
    if num_targets is None:
        nts = np.zeros_like(lengths)
    else:
        nts = np.asarray(num_targets, dtype=np.int64)
    return int(sum(attn_pairs_per_seq(L, n, local_window, global_window) for L, n in zip(lengths, nts)))


def attn_fwd_flops(pairs: float, num_heads: int, d_qk: int, d_v: int) -> float:
    return 2.0 * (d_qk + d_v) * pairs * num_heads


def attn_bwd_flops(pairs: float, num_heads: int, d_qk: int, d_v: int) -> float:
    # recompute S (d_qk), dP = dO V^T (d_v), dV = P^T dO (d_v), dQ, dK (d_qk each)
    return 2.0 * (3 * d_qk + 2 * d_v) * pairs * num_heads


def f1_flops(tokens: int, d_model: int, num_heads: int, d_qk: int, d_v: int) -> float:
    return 2.0 * tokens * d_model * num_heads * (2 * d_qk + 2 * d_v)


def f2_flops(tokens: int, d_model: int, num_heads: int, d_v: int, width_factor: int = 1) -> float:
    return 2.0 * tokens * width_factor * num_heads * d_v * d_model


def gate_bytes(tokens: int, num_heads: int, d_v: int, elem_bytes: int = 2) -> float:
    """LayerNorm(O) * U: read O and U, write G (one pass each)."""
    return 3.0 * tokens * num_heads * d_v * elem_bytes


def layer_bwd_gemm_flops(T: int, d_model: int, num_heads: int, d_qk: int, d_v: int) -> float:
    """Algorithmic FLOPs of the layer backward's GEMMs, twice the forward's (the
    DLRMv4 page's Table 7 counts forward + backward as three times the forward):
    dG = dY W2^T, dW2 = G^T dY (2 T D H d_v each), dX = dZ W1^T, dW1 = X^T dZ
    (2 T D W each).  A recompute of the pre-activation X W1 is not counted."""
    hv = num_heads * d_v
    width = num_heads * (2 * d_v + 2 * d_qk)
    return 2.0 * T * (2 * d_model * hv + 2 * d_model * width)



def truncate_bytes(kept_tokens: int, row_bytes: int, num_seqs: int) -> float:
    """Attention-truncation gather: read and write each kept row once, plus the
    two offset arrays."""
    return 2.0 * kept_tokens * row_bytes + 2.0 * 8 * (num_seqs + 1)
