"""CPU oracle for HSTU jagged attention and the transduction layer (fp64).

TEST INFRASTRUCTURE ONLY.  The library and its binding never import this
package; only `tests/`, the smoke check in `__graft_entry__` and the CPU
baseline leg of `bench.py` may.  It shares no code with the CUDA path.

The arithmetic lives in `hstu_oracle.c` (plain loops, double accumulation);
this module builds it with gcc when needed and marshals numpy arrays.
Inputs in bf16 are widened exactly to float64 before the call.

Pins (tests/test_oracle_pins.py): a hand-worked three-token example, a dense
brute-force formulation, torch float64 autograd, central finite differences,
causality / independence / linearity invariants, the exhaustive bucket check,
the cost formulas of the DLRMv4 page's Table 7, and for the truncation gather
a hand-worked batch and its equivalence with a local attention window.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_time_bucket.restype = ctypes.c_int
            lib.oracle_time_bucket.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
            lib.oracle_pos_index.restype = ctypes.c_int
            lib.oracle_pos_index.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int]
            lib.oracle_visible.restype = ctypes.c_int
            lib.oracle_visible.argtypes = [ctypes.c_int64] * 4
            lib.oracle_visible_sl.restype = ctypes.c_int
            lib.oracle_visible_sl.argtypes = [ctypes.c_int64] * 6
            lib.oracle_set_windows.restype = None
            lib.oracle_set_windows.argtypes = [ctypes.c_int64] * 2
            lib.oracle_set_variants.restype = None
            lib.oracle_set_variants.argtypes = [ctypes.c_int64] * 2
            _lib = lib
    return _lib


def default_threads() -> int:
    return int(os.environ.get("HSTU_ORACLE_THREADS", os.cpu_count() or 1))


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (any float dtype): widen exactly
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i64(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _i32_or_none(a):
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _p(a, kind):
    if a is None:
        return ctypes.cast(None, kind)
    return a.ctypes.data_as(kind)


def time_bucket(t_i: int, t_j: int, num_buckets: int) -> int:
    return _load().oracle_time_bucket(int(t_i), int(t_j), int(num_buckets))


def pos_index(p_i: int, p_j: int, pos_lo: int, pos_hi: int) -> int:
    return _load().oracle_pos_index(int(p_i), int(p_j), int(pos_lo), int(pos_hi))


def visible(i: int, j: int, L: int, n_t: int) -> bool:
    return bool(_load().oracle_visible(int(i), int(j), int(L), int(n_t)))


def visible_sl(i: int, j: int, L: int, n_t: int, local_window: int, global_window: int) -> bool:
    """visible() restricted to the semi-local windows (local_window <= 0: no restriction)."""
    return bool(_load().oracle_visible_sl(int(i), int(j), int(L), int(n_t), int(local_window),
                                          int(global_window)))


def bias_pair_counts(seq_offsets, timestamps, num_targets, pos_lo, pos_hi, num_buckets,
                     local_window=0, global_window=0, threads=None, cand_own_index=False):
    """Visible pairs per rab_pos entry and per rab_time bucket, one head (int64
    arrays [pos_hi - pos_lo + 1] and [num_buckets]), with the attention's own
    visibility rule, windows and index functions."""
    off, ts, nt = _i64(seq_offsets), _i64(timestamps), _i32_or_none(num_targets)
    pc = np.zeros(int(pos_hi) - int(pos_lo) + 1, dtype=np.int64)
    tc = np.zeros(int(num_buckets), dtype=np.int64)
    with _Windows(0, 0, cand_own_index, False):
        _load().oracle_bias_pair_counts(ctypes.c_int(len(off) - 1), _p(off, _i64p), _p(nt, _i32p), _p(ts, _i64p),
                                        ctypes.c_int(int(pos_lo)), ctypes.c_int(int(pos_hi)),
                                        ctypes.c_int(int(num_buckets)), ctypes.c_int64(int(local_window)),
                                        ctypes.c_int64(int(global_window)), _p(pc, _i64p), _p(tc, _i64p),
                                        ctypes.c_int(threads or default_threads()))
    return pc, tc


class _Windows:
    """Readings applied by the oracle's attention for the duration of one call: the
    semi-local windows, candidates at their own index instead of the shared slot
    after the history, and one pair of bias tables per head instead of a shared pair."""

    def __init__(self, local_window=0, global_window=0, cand_own_index=False, per_head_tables=False):
        self.w = (int(local_window), int(global_window))
        self.v = (int(bool(cand_own_index)), int(bool(per_head_tables)))

    def __enter__(self):
        _load().oracle_set_windows(ctypes.c_int64(self.w[0]), ctypes.c_int64(self.w[1]))
        _load().oracle_set_variants(ctypes.c_int64(self.v[0]), ctypes.c_int64(self.v[1]))

    def __exit__(self, *exc):
        _load().oracle_set_windows(ctypes.c_int64(0), ctypes.c_int64(0))
        _load().oracle_set_variants(ctypes.c_int64(0), ctypes.c_int64(0))


def _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi):
    """(rab_pos, rab_time) flattened to float64, the bucket count, and whether the
    tables are per head: 1-D tables are shared by the heads, 2-D ones are
    [num_heads, entries]."""
    rp, rt = np.asarray(rab_pos), np.asarray(rab_time)
    if hasattr(rab_pos, "detach"):
        rp = rab_pos.detach().cpu().double().numpy()
    if hasattr(rab_time, "detach"):
        rt = rab_time.detach().cpu().double().numpy()
    per_head = rp.ndim == 2
    assert rt.ndim == rp.ndim and (not per_head or (rp.shape[0] == rt.shape[0] == num_heads))
    assert rp.shape[-1] == int(pos_hi) - int(pos_lo) + 1
    return (np.ascontiguousarray(rp, dtype=np.float64).reshape(-1), np.ascontiguousarray(rt, dtype=np.float64).reshape(-1),
            rt.shape[-1], per_head)


class _Attn:
    """Marshalled common attention arguments."""

    def __init__(self, seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time,
                 pos_lo, pos_hi, inv_n):
        self.off = _i64(seq_offsets)
        self.ts = _i64(timestamps)
        self.nt = _i32_or_none(num_targets)
        self.B = len(self.off) - 1
        self.T = int(self.off[-1]) if self.B >= 0 else 0
        self.q, self.k, self.v = _f64(q), _f64(k), _f64(v)
        self.H = self.q.shape[1]
        self.dqk = self.q.shape[2]
        self.dv = self.v.shape[2]
        self.lo, self.hi = int(pos_lo), int(pos_hi)
        self.rp, self.rt, self.nb, self.per_head = _tables(rab_pos, rab_time, self.H, self.lo, self.hi)
        self.table_shapes = (np.shape(rab_pos), np.shape(rab_time))
        self.inv_n = float(inv_n)

    def head(self):
        return [ctypes.c_int(self.B), _p(self.off, _i64p), _p(self.nt, _i32p), ctypes.c_int(self.H),
                ctypes.c_int(self.dqk), ctypes.c_int(self.dv), _p(self.q, _f64p), _p(self.k, _f64p),
                _p(self.v, _f64p), _p(self.ts, _i64p), _p(self.rp, _f64p), ctypes.c_int(self.lo),
                ctypes.c_int(self.hi), _p(self.rt, _f64p), ctypes.c_int(self.nb),
                ctypes.c_double(self.inv_n)]


def attn_fwd(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi,
             inv_n, threads=None, local_window=0, global_window=0, cand_own_index=False):
    """O[T, H, dv] of the jagged SiLU attention (float64).  Tables [H, entries]
    are per head; cand_own_index puts each candidate at its own index."""
    a = _Attn(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n)
    out = np.zeros((a.T, a.H, a.dv), dtype=np.float64)
    with _Windows(local_window, global_window, cand_own_index, a.per_head):
        _load().oracle_attn_fwd(*a.head(), _p(out, _f64p), ctypes.c_int(threads or default_threads()))
    return out


def attn_fwd_rows(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo,
                  pos_hi, inv_n, rows, threads=None, local_window=0, global_window=0, cand_own_index=False):
    """O rows for the given global token indices: [n, H, dv]."""
    a = _Attn(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n)
    rows = _i64(rows)
    out = np.zeros((len(rows), a.H, a.dv), dtype=np.float64)
    with _Windows(local_window, global_window, cand_own_index, a.per_head):
        _load().oracle_attn_fwd_rows(*a.head(), ctypes.c_int64(len(rows)), _p(rows, _i64p),
                                     _p(out, _f64p), ctypes.c_int(threads or default_threads()))
    return out


def attn_bwd(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi,
             inv_n, dout, threads=None, local_window=0, global_window=0, cand_own_index=False):
    """(dq, dk, dv, d_rab_pos, d_rab_time) for the loss sum(O * dout); the table
    gradients have the tables' shapes (per head for [H, entries] tables)."""
    a = _Attn(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n)
    do = _f64(dout)
    dq = np.zeros_like(a.q)
    dk = np.zeros_like(a.k)
    dv = np.zeros_like(a.v)
    drp = np.zeros_like(a.rp)
    drt = np.zeros_like(a.rt)
    with _Windows(local_window, global_window, cand_own_index, a.per_head):
        _load().oracle_attn_bwd(*a.head(), _p(do, _f64p), _p(dq, _f64p), _p(dk, _f64p), _p(dv, _f64p),
                                _p(drp, _f64p), _p(drt, _f64p), ctypes.c_int(threads or default_threads()))
    return dq, dk, dv, drp.reshape(a.table_shapes[0]), drt.reshape(a.table_shapes[1])


def attn_bwd_rows(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo,
                  pos_hi, inv_n, dout, q_rows, k_rows, threads=None, local_window=0, global_window=0,
                  cand_own_index=False):
    """dq for query rows `q_rows`; dk, dv for key rows `k_rows`."""
    a = _Attn(seq_offsets, timestamps, num_targets, q, k, v, rab_pos, rab_time, pos_lo, pos_hi, inv_n)
    do = _f64(dout)
    qr, kr = _i64(q_rows), _i64(k_rows)
    dq = np.zeros((len(qr), a.H, a.dqk))
    dk = np.zeros((len(kr), a.H, a.dqk))
    dv = np.zeros((len(kr), a.H, a.dv))
    with _Windows(local_window, global_window, cand_own_index, a.per_head):
        _load().oracle_attn_bwd_rows(*a.head(), _p(do, _f64p), ctypes.c_int64(len(qr)), _p(qr, _i64p),
                                     _p(dq, _f64p), ctypes.c_int64(len(kr)), _p(kr, _i64p),
                                     _p(dk, _f64p), _p(dv, _f64p),
                                     ctypes.c_int(threads or default_threads()))
    return dq, dk, dv


def linear(x, w, bias=None, apply_silu=False, threads=None):
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    T, m = x.shape
    n = w.shape[1]
    out = np.zeros((T, n))
    _load().oracle_linear(ctypes.c_int64(T), ctypes.c_int(m), ctypes.c_int(n), _p(x, _f64p),
                          _p(w, _f64p), _p(bias, _f64p), ctypes.c_int(int(apply_silu)),
                          _p(out, _f64p), ctypes.c_int(threads or default_threads()))
    return out


def norm_gate(o, u, gamma, beta, eps=1e-5, threads=None):
    o, u, gamma, beta = _f64(o), _f64(u), _f64(gamma), _f64(beta)
    T, F = o.shape
    g = np.zeros((T, F))
    _load().oracle_norm_gate(ctypes.c_int64(T), ctypes.c_int(F), _p(o, _f64p), _p(u, _f64p),
                             _p(gamma, _f64p), _p(beta, _f64p), ctypes.c_double(eps), _p(g, _f64p),
                             ctypes.c_int(threads or default_threads()))
    return g


def layer_fwd(seq_offsets, timestamps, num_targets, x, w1, b1, w2, b2, ln_gamma, ln_beta,
              rab_pos, rab_time, pos_lo, pos_hi, inv_n, num_heads, d_qk, d_v, ln_eps=1e-5,
              threads=None, want_intermediates=False, out_cat=False, local_window=0, global_window=0,
              cand_own_index=False):
    """Y[T, D] of one transduction layer (and optionally uvqk, O).  out_cat: the
    output projection reads [U | O | G] (W2 is [3 H d_v, D]) instead of G;
    local_window / global_window: semi-local attention (see visible_sl)."""
    off, ts, nt = _i64(seq_offsets), _i64(timestamps), _i32_or_none(num_targets)
    x, w1, b1, w2, b2 = _f64(x), _f64(w1), _f64(b1), _f64(w2), _f64(b2)
    g, be = _f64(ln_gamma), _f64(ln_beta)
    rp, rt, nb, per_head = _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi)
    T, D = x.shape
    W = num_heads * (2 * d_v + 2 * d_qk)
    assert w2.shape == ((3 if out_cat else 1) * num_heads * d_v, D)
    y = np.zeros((T, D))
    uvqk = np.zeros((T, W)) if want_intermediates else None
    o = np.zeros((T, num_heads * d_v)) if want_intermediates else None
    with _Windows(local_window, global_window, cand_own_index, per_head):
        _layer_fwd_call(off, nt, num_heads, d_qk, d_v, D, x, w1, b1, w2, b2, g, be, ln_eps, ts, rp, pos_lo,
                        pos_hi, rt, nb, inv_n, y, uvqk, o, out_cat, threads)
    if want_intermediates:
        return y, uvqk, o
    return y


def _layer_fwd_call(off, nt, num_heads, d_qk, d_v, D, x, w1, b1, w2, b2, g, be, ln_eps, ts, rp, pos_lo, pos_hi,
                    rt, nb, inv_n, y, uvqk, o, out_cat, threads):
    _load().oracle_layer_fwd(
        ctypes.c_int(len(off) - 1), _p(off, _i64p), _p(nt, _i32p), ctypes.c_int(num_heads),
        ctypes.c_int(d_qk), ctypes.c_int(d_v), ctypes.c_int(D), _p(x, _f64p), _p(w1, _f64p),
        _p(b1, _f64p), _p(w2, _f64p), _p(b2, _f64p), _p(g, _f64p), _p(be, _f64p),
        ctypes.c_double(ln_eps), _p(ts, _i64p), _p(rp, _f64p), ctypes.c_int(int(pos_lo)),
        ctypes.c_int(int(pos_hi)), _p(rt, _f64p), ctypes.c_int(int(nb)), ctypes.c_double(inv_n),
        _p(y, _f64p), _p(uvqk, _f64p), _p(o, _f64p), ctypes.c_int(int(out_cat)),
        ctypes.c_int(threads or default_threads()))


def layer_bwd(seq_offsets, timestamps, num_targets, x, w1, b1, w2, ln_gamma, ln_beta, rab_pos, rab_time,
              pos_lo, pos_hi, inv_n, num_heads, d_qk, d_v, dy, ln_eps=1e-5, threads=None, out_cat=False,
              local_window=0, global_window=0, cand_own_index=False):
    """Gradients of sum(Y * dy) for one transduction layer: a dict with dx, dw1, db1,
    dw2, db2, d_ln_gamma, d_ln_beta, d_rab_pos, d_rab_time (out_cat as in layer_fwd)."""
    off, ts, nt = _i64(seq_offsets), _i64(timestamps), _i32_or_none(num_targets)
    x, w1, b1, w2 = _f64(x), _f64(w1), _f64(b1), _f64(w2)
    g, be, dyy = _f64(ln_gamma), _f64(ln_beta), _f64(dy)
    rp, rt, nb, per_head = _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi)
    T, D = x.shape
    hv = num_heads * d_v
    W = num_heads * (2 * d_v + 2 * d_qk)
    F = (3 if out_cat else 1) * hv
    assert w2.shape == (F, D)
    out = {"dx": np.zeros((T, D)), "dw1": np.zeros((D, W)), "db1": np.zeros(W), "dw2": np.zeros((F, D)),
           "db2": np.zeros(D), "d_ln_gamma": np.zeros(hv), "d_ln_beta": np.zeros(hv),
           "d_rab_pos": np.zeros(len(rp)), "d_rab_time": np.zeros(len(rt))}
    with _Windows(local_window, global_window, cand_own_index, per_head):
        _layer_bwd_call(off, nt, num_heads, d_qk, d_v, D, x, w1, b1, w2, g, be, ln_eps, ts, rp, pos_lo, pos_hi,
                        rt, nb, inv_n, dyy, out, out_cat, threads)
    out["d_rab_pos"] = out["d_rab_pos"].reshape(np.shape(rab_pos))
    out["d_rab_time"] = out["d_rab_time"].reshape(np.shape(rab_time))
    return out


def _layer_bwd_call(off, nt, num_heads, d_qk, d_v, D, x, w1, b1, w2, g, be, ln_eps, ts, rp, pos_lo, pos_hi, rt,
                    nb, inv_n, dyy, out, out_cat, threads):
    _load().oracle_layer_bwd(
        ctypes.c_int(len(off) - 1), _p(off, _i64p), _p(nt, _i32p), ctypes.c_int(num_heads),
        ctypes.c_int(d_qk), ctypes.c_int(d_v), ctypes.c_int(D), _p(x, _f64p), _p(w1, _f64p),
        _p(b1, _f64p), _p(w2, _f64p), _p(g, _f64p), _p(be, _f64p), ctypes.c_double(ln_eps),
        _p(ts, _i64p), _p(rp, _f64p), ctypes.c_int(int(pos_lo)), ctypes.c_int(int(pos_hi)), _p(rt, _f64p),
        ctypes.c_int(int(nb)), ctypes.c_double(inv_n), _p(dyy, _f64p), _p(out["dx"], _f64p),
        _p(out["dw1"], _f64p), _p(out["db1"], _f64p), _p(out["dw2"], _f64p), _p(out["db2"], _f64p),
        _p(out["d_ln_gamma"], _f64p), _p(out["d_ln_beta"], _f64p), _p(out["d_rab_pos"], _f64p),
        _p(out["d_rab_time"], _f64p), ctypes.c_int(int(out_cat)), ctypes.c_int(threads or default_threads()))


def attn_inputs_fwd(inp, threads=None):
    """Oracle forward over a `workloads.AttnInputs`-like object."""
    return attn_fwd(inp.seq_offsets, inp.timestamps, inp.num_targets, inp.q, inp.k, inp.v,
                    inp.rab_pos, inp.rab_time, inp.pos_lo, inp.pos_hi, inp.inv_n, threads)


def jagged_truncate(seq_offsets, num_targets, keep, rows):
    """Attention truncation (the ULTRA-HSTU review in the pages): after the
    first layers over whole histories, later layers run only over a segment
    of each history, its most recent events.  Reading: a sequence keeps its
    last min(hist, keep) history tokens and all of its candidates, in order;
    `rows` is any per-token array (layer activations, timestamps).  Returns
    (new seq_offsets, kept rows).  Plain per-sequence slicing."""
    off = np.asarray(seq_offsets, dtype=np.int64)
    B = len(off) - 1
    nt = np.zeros(B, np.int64) if num_targets is None else np.asarray(num_targets, np.int64)
    rows = np.asarray(rows)
    new_off = [0]
    pieces = []
    for b in range(B):
        start, end = int(off[b]), int(off[b + 1])
        hist = end - start - int(nt[b])
        first = start + hist - min(hist, int(keep))   # first kept history token
        pieces.append(rows[first:end])
        new_off.append(new_off[-1] + (end - first))
    kept = np.concatenate(pieces) if pieces else rows[:0]
    return np.asarray(new_off, dtype=np.int64), kept
