"""Python binding of libhstu (ctypes): argument marshalling only.

Every function here has the name of the C entry point it calls (include/hstu.h)
and does no arithmetic of the method: it checks tensor placement, allocates
outputs and workspace through PyTorch's allocator, and passes raw device
pointers plus the current CUDA stream.  There is no fallback: if the library
cannot be loaded or built, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading
from typing import Optional

import torch

from . import build as _build

HSTU_F32, HSTU_BF16 = 0, 1
# hstu_attn_desc.debug_checks: the bounded-wait test hook (see include/hstu.h)
HSTU_DEBUG_WAIT_TEST = 2
STATUS = {0: "HSTU_OK", 1: "HSTU_ERR_INVALID_ARG", 2: "HSTU_ERR_UNSUPPORTED", 3: "HSTU_ERR_WORKSPACE",
          4: "HSTU_ERR_CUDA", 5: "HSTU_ERR_DEVICE_CHECK"}

EXPORTED = ["hstu_status_string", "hstu_version", "hstu_attn_workspace_size",
            "hstu_layer_workspace_size", "hstu_attn_fwd", "hstu_attn_bwd", "hstu_layer_fwd",
            "hstu_check_device_flag", "hstu_debug_bias_indices", "hstu_debug_schedule",
            "hstu_attn_fwd_noalloc", "hstu_layer_bwd_workspace_size", "hstu_layer_bwd",
            "hstu_jagged_truncate", "hstu_quantize_weight_e4m3", "hstu_quantize_rows_e4m3", "hstu_gemm_e4m3",
            "hstu_e4m3_weight_bytes"]


class HstuError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class hstu_attn_desc(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
                ("total_tokens", ctypes.c_int64), ("num_heads", ctypes.c_int32),
                ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("inv_n", ctypes.c_float), ("pos_lo", ctypes.c_int32), ("pos_hi", ctypes.c_int32),
                ("num_time_buckets", ctypes.c_int32), ("debug_checks", ctypes.c_int32),
                ("local_window", ctypes.c_int32), ("global_window", ctypes.c_int32), ("fp8_qk", ctypes.c_int32),
                ("cand_positions", ctypes.c_int32), ("per_head_tables", ctypes.c_int32)]


class hstu_layer_desc(ctypes.Structure):
    _fields_ = [("attn", hstu_attn_desc), ("d_model", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("output_concat", ctypes.c_int32), ("fp8_projections", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB


def load_library(allow_build: bool = True) -> ctypes.CDLL:
    """Load libhstu.so, compiling it first when it is missing or stale."""
    global _lib
    with _lock:
        if _lib is None:
            if allow_build and _build.needs_build():
                _build.build()
            if not os.path.exists(_build.LIB):
                raise RuntimeError(f"libhstu.so not found at {_build.LIB}; build it with "
                                   "python -m hstu_sequential_transduction_b200.build")
            lib = ctypes.CDLL(_build.LIB)
            lib.hstu_status_string.restype = ctypes.c_char_p
            lib.hstu_status_string.argtypes = [ctypes.c_int]
            lib.hstu_version.restype = ctypes.c_int
            for name in EXPORTED[2:]:
                getattr(lib, name).restype = ctypes.c_int
            lib.hstu_e4m3_weight_bytes.restype = ctypes.c_size_t
            lib.hstu_e4m3_weight_bytes.argtypes = [ctypes.c_int32, ctypes.c_int32]
            _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != 0:
        raise HstuError(fn, status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HSTU_BF16
    if t.dtype == torch.float32:
        return HSTU_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def make_attn_desc(num_seqs, max_seq_len, total_tokens, num_heads, d_qk, d_v, dtype, inv_n,
                   pos_lo, pos_hi, num_time_buckets, local_window=0, global_window=0,
                   fp8_qk=False, cand_own_index=False, per_head_tables=False) -> hstu_attn_desc:
    return hstu_attn_desc(int(num_seqs), int(max_seq_len), int(total_tokens), int(num_heads),
                          int(d_qk), int(d_v), int(dtype), float(inv_n), int(pos_lo), int(pos_hi),
                          int(num_time_buckets), 0, int(local_window), int(global_window), int(bool(fp8_qk)),
                          int(bool(cand_own_index)), int(bool(per_head_tables)))


def hstu_status_string(status: int) -> str:
    return load_library().hstu_status_string(int(status)).decode()


def hstu_version() -> int:
    return load_library().hstu_version()


def hstu_attn_workspace_size(desc: hstu_attn_desc, is_bwd: bool) -> int:
    n = ctypes.c_size_t(0)
    _check("hstu_attn_workspace_size",
           load_library().hstu_attn_workspace_size(ctypes.byref(desc), int(is_bwd), ctypes.byref(n)))
    return n.value


def hstu_layer_workspace_size(desc: hstu_layer_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("hstu_layer_workspace_size",
           load_library().hstu_layer_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi):
    """(num_time_buckets, per_head) of a pair of bias tables: both 1-D (shared by
    the heads) or both [num_heads, n] (one row per head)."""
    npos = int(pos_hi) - int(pos_lo) + 1
    if rab_pos.dim() != rab_time.dim() or rab_pos.dim() not in (1, 2):
        raise ValueError("rab_pos and rab_time must both be 1-D or both [num_heads, n]")
    per_head = rab_pos.dim() == 2
    if per_head and (rab_pos.shape[0] != num_heads or rab_time.shape[0] != num_heads):
        raise ValueError(f"per-head tables need {num_heads} rows")
    if rab_pos.shape[-1] != npos:
        raise ValueError(f"rab_pos has {rab_pos.shape[-1]} entries for distances {pos_lo}..{pos_hi}")
    return rab_time.shape[-1], per_head


def _attn_desc_from(q, v, seq_offsets, max_seq_len, inv_n, pos_lo, pos_hi, rab_pos, rab_time, local_window=0,
                    global_window=0, fp8_qk=False, cand_own_index=False):
    nb, per_head = _tables(rab_pos, rab_time, q.shape[1], pos_lo, pos_hi)
    return make_attn_desc(seq_offsets.numel() - 1, max_seq_len, q.shape[0], q.shape[1], q.shape[2],
                          v.shape[2], _dtype_code(q), inv_n, pos_lo, pos_hi, nb, local_window,
                          global_window, fp8_qk, cand_own_index, per_head)


def hstu_attn_fwd(q, k, v, seq_offsets, timestamps, num_targets, rab_pos, rab_time, *,
                  max_seq_len: int, inv_n: float, pos_lo: int, pos_hi: int, out=None,
                  workspace=None, stream=None, local_window: int = 0, global_window: int = 0,
                  fp8_qk: bool = False, cand_own_index: bool = False):
    """O = jagged SiLU attention; q, k [T, H, d_qk], v [T, H, d_v] on CUDA.
    local_window > 0 applies the semi-local mask; fp8_qk computes Q K^T on E4M3
    codes of q and k; cand_own_index puts candidate i at position i; 2-D tables
    [H, n] give each head its own (see hstu_attn_desc)."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        _dev(t, name, q.dtype)
    _dev(seq_offsets, "seq_offsets", torch.int64)
    _dev(timestamps, "timestamps", torch.int64)
    _dev(num_targets, "num_targets", torch.int32)
    _dev(rab_pos, "rab_pos", torch.float32)
    _dev(rab_time, "rab_time", torch.float32)
    desc = _attn_desc_from(q, v, seq_offsets, max_seq_len, inv_n, pos_lo, pos_hi, rab_pos, rab_time, local_window,
                           global_window, fp8_qk, cand_own_index)
    if out is None:
        out = torch.empty_like(v)
    _dev(out, "out", q.dtype)
    need = hstu_attn_workspace_size(desc, False)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    _check("hstu_attn_fwd", load_library().hstu_attn_fwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(timestamps),
        _ptr(num_targets), _ptr(rab_pos), _ptr(rab_time), _ptr(out), _ptr(workspace),
        ctypes.c_size_t(workspace.numel()), _stream(stream)))
    return out


def hstu_attn_fwd_noalloc(q, k, v, seq_offsets, timestamps, num_targets, rab_pos, rab_time, out,
                          *, max_seq_len: int, inv_n: float, pos_lo: int, pos_hi: int, stream=None,
                          cand_own_index: bool = False):
    """hstu_attn_fwd without a workspace: the library keeps the scheduler's
    scratch in a static device array (for callers that cannot allocate).
    `out` must be preallocated; nothing is allocated here either."""
    desc = _attn_desc_from(q, v, seq_offsets, max_seq_len, inv_n, pos_lo, pos_hi, rab_pos, rab_time,
                           cand_own_index=cand_own_index)
    _check("hstu_attn_fwd_noalloc", load_library().hstu_attn_fwd_noalloc(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(timestamps),
        _ptr(num_targets), _ptr(rab_pos), _ptr(rab_time), _ptr(out), _stream(stream)))
    return out


def hstu_attn_bwd(q, k, v, seq_offsets, timestamps, num_targets, rab_pos, rab_time, dout, *,
                  max_seq_len: int, inv_n: float, pos_lo: int, pos_hi: int, grads=None,
                  workspace=None, stream=None, local_window: int = 0, global_window: int = 0,
                  cand_own_index: bool = False):
    """(dq, dk, dv, d_rab_pos, d_rab_time) for the loss sum(O * dout); the table
    gradients have the tables' shapes."""
    for name, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _dev(t, name, q.dtype)
    _dev(seq_offsets, "seq_offsets", torch.int64)
    _dev(timestamps, "timestamps", torch.int64)
    _dev(num_targets, "num_targets", torch.int32)
    desc = _attn_desc_from(q, v, seq_offsets, max_seq_len, inv_n, pos_lo, pos_hi, rab_pos, rab_time, local_window,
                           global_window, cand_own_index=cand_own_index)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(rab_pos), torch.empty_like(rab_time))
    dq, dk, dv, drp, drt = grads
    need = hstu_attn_workspace_size(desc, True)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    _check("hstu_attn_bwd", load_library().hstu_attn_bwd(
        ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(timestamps),
        _ptr(num_targets), _ptr(rab_pos), _ptr(rab_time), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(drp), _ptr(drt), _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream)))
    return dq, dk, dv, drp, drt


def hstu_layer_fwd(x, w1, b1, w2, b2, ln_gamma, ln_beta, seq_offsets, timestamps, num_targets,
                   rab_pos, rab_time, *, num_heads: int, d_qk: int, d_v: int, max_seq_len: int,
                   inv_n: float, pos_lo: int, pos_hi: int, ln_eps: float = 1e-5, y=None,
                   saved_uvqk=None, saved_o=None, workspace=None, stream=None, output_concat: bool = False,
                   fp8_projections: bool = False, local_window: int = 0, global_window: int = 0,
                   cand_own_index: bool = False):
    """Y = f2(LayerNorm(attention(SiLU(f1(X)))) * U) for one layer; with
    output_concat, f2 reads [U | O | G] and w2 is [3 H d_v, D]; with
    fp8_projections, w1 and w2 are E4M3 weight packs (quantize_weight_e4m3)."""
    for name, t in (("x", x), ("b1", b1), ("b2", b2)) + (() if fp8_projections else (("w1", w1), ("w2", w2))):
        _dev(t, name, x.dtype)
    if fp8_projections:
        _dev(w1, "w1", torch.uint8)
        _dev(w2, "w2", torch.uint8)
    _dev(ln_gamma, "ln_gamma", torch.float32)
    _dev(ln_beta, "ln_beta", torch.float32)
    T, D = x.shape
    nb, per_head = _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi)
    attn = make_attn_desc(seq_offsets.numel() - 1, max_seq_len, T, num_heads, d_qk, d_v,
                          _dtype_code(x), inv_n, pos_lo, pos_hi, nb, local_window, global_window,
                          False, cand_own_index, per_head)
    desc = hstu_layer_desc(attn, int(D), float(ln_eps), int(bool(output_concat)), int(bool(fp8_projections)))
    if fp8_projections:
        W = num_heads * (2 * d_v + 2 * d_qk)
        for name, t, k, n in (("w1", w1, D, W), ("w2", w2, num_heads * d_v, D)):
            if t.numel() < hstu_e4m3_weight_bytes(k, n):
                raise ValueError(f"{name} is not an E4M3 pack of a [{k}, {n}] weight")
    elif w2.shape[0] != (3 if output_concat else 1) * num_heads * d_v:
        raise ValueError(f"w2 has {w2.shape[0]} rows for output_concat={output_concat}")
    if y is None:
        y = torch.empty((T, D), dtype=x.dtype, device=x.device)
    if workspace is None:
        workspace = alloc_workspace(hstu_layer_workspace_size(desc), x.device)
    _check("hstu_layer_fwd", load_library().hstu_layer_fwd(
        ctypes.byref(desc), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(ln_gamma),
        _ptr(ln_beta), _ptr(seq_offsets), _ptr(timestamps), _ptr(num_targets), _ptr(rab_pos),
        _ptr(rab_time), _ptr(y), _ptr(saved_uvqk), _ptr(saved_o), _ptr(workspace),
        ctypes.c_size_t(workspace.numel()), _stream(stream)))
    return y


def hstu_layer_bwd_workspace_size(desc: hstu_layer_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("hstu_layer_bwd_workspace_size",
           load_library().hstu_layer_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return n.value


def hstu_layer_bwd(x, w1, b1, w2, ln_gamma, ln_beta, seq_offsets, timestamps, num_targets, rab_pos, rab_time,
                   saved_uvqk, saved_o, dy, *, num_heads: int, d_qk: int, d_v: int, max_seq_len: int,
                   inv_n: float, pos_lo: int, pos_hi: int, ln_eps: float = 1e-5, workspace=None, stream=None,
                   output_concat: bool = False, local_window: int = 0, global_window: int = 0,
                   cand_own_index: bool = False):
    """Gradients of sum(Y * dy) for one layer (bf16): a dict with dx (bf16) and the
    float32 parameter gradients dw1, db1, dw2, db2, d_ln_gamma, d_ln_beta,
    d_rab_pos, d_rab_time (the tables' shapes; output_concat as in hstu_layer_fwd)."""
    for name, t in (("x", x), ("w1", w1), ("b1", b1), ("w2", w2), ("saved_uvqk", saved_uvqk),
                    ("saved_o", saved_o), ("dy", dy)):
        _dev(t, name, x.dtype)
    _dev(ln_gamma, "ln_gamma", torch.float32)
    _dev(ln_beta, "ln_beta", torch.float32)
    T, D = x.shape
    W = w1.shape[1]
    hv = num_heads * d_v
    nb, per_head = _tables(rab_pos, rab_time, num_heads, pos_lo, pos_hi)
    attn = make_attn_desc(seq_offsets.numel() - 1, max_seq_len, T, num_heads, d_qk, d_v,
                          _dtype_code(x), inv_n, pos_lo, pos_hi, nb, local_window, global_window,
                          False, cand_own_index, per_head)
    desc = hstu_layer_desc(attn, int(D), float(ln_eps), int(bool(output_concat)))
    F = (3 if output_concat else 1) * hv
    if w2.shape[0] != F:
        raise ValueError(f"w2 has {w2.shape[0]} rows for output_concat={output_concat}")
    dev = x.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty((T, D), dtype=x.dtype, device=dev), "dw1": torch.empty((D, W), **f32),
           "db1": torch.empty(W, **f32), "dw2": torch.empty((F, D), **f32), "db2": torch.empty(D, **f32),
           "d_ln_gamma": torch.empty(hv, **f32), "d_ln_beta": torch.empty(hv, **f32),
           "d_rab_pos": torch.empty(rab_pos.shape, **f32), "d_rab_time": torch.empty(rab_time.shape, **f32)}
    if workspace is None:
        workspace = alloc_workspace(hstu_layer_bwd_workspace_size(desc), dev)
    _check("hstu_layer_bwd", load_library().hstu_layer_bwd(
        ctypes.byref(desc), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(ln_gamma), _ptr(ln_beta),
        _ptr(seq_offsets), _ptr(timestamps), _ptr(num_targets), _ptr(rab_pos), _ptr(rab_time),
        _ptr(saved_uvqk), _ptr(saved_o), _ptr(dy), _ptr(out["dx"]), _ptr(out["dw1"]), _ptr(out["db1"]),
        _ptr(out["dw2"]), _ptr(out["db2"]), _ptr(out["d_ln_gamma"]), _ptr(out["d_ln_beta"]),
        _ptr(out["d_rab_pos"]), _ptr(out["d_rab_time"]), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
        _stream(stream)))
    return out


def hstu_e4m3_weight_bytes(K: int, N: int) -> int:
    return int(load_library().hstu_e4m3_weight_bytes(int(K), int(N)))


def quantize_weight_e4m3(w, stream=None):
    """E4M3 weight pack of a bf16 weight w [K, N]: uint8 tensor holding the
    codes [N, K] and, from byte align256(N K), the float32 scales [N]."""
    _dev(w, "w", torch.bfloat16)
    K, N = w.shape
    pack = torch.empty(hstu_e4m3_weight_bytes(K, N), dtype=torch.uint8, device=w.device)
    _check("hstu_quantize_weight_e4m3", load_library().hstu_quantize_weight_e4m3(
        _ptr(w), ctypes.c_int32(K), ctypes.c_int32(N), _ptr(pack), _stream(stream)))
    return pack


def e4m3_pack_parts(pack, K: int, N: int):
    """(codes [N, K] uint8, scales [N] float32) views of a weight pack."""
    off = (N * K + 255) // 256 * 256
    return pack[:N * K].view(N, K), pack[off:off + 4 * N].view(torch.float32)


def quantize_rows_e4m3(x, stream=None):
    """Per-row E4M3 codes [R, K] (uint8) and scales [R] (float32) of a bf16 x [R, K]."""
    _dev(x, "x", torch.bfloat16)
    R, K = x.shape
    codes = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty(R, dtype=torch.float32, device=x.device)
    _check("hstu_quantize_rows_e4m3", load_library().hstu_quantize_rows_e4m3(
        _ptr(x), ctypes.c_int64(R), ctypes.c_int32(K), _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def gemm_e4m3(codes, scales, wpack, N: int, bias=None, apply_silu: bool = False, y=None, workspace=None,
              stream=None):
    """bf16 y [M, N] = dequant(codes, scales) dequant(W)^T + bias (optionally SiLU)."""
    _dev(codes, "codes", torch.uint8)
    _dev(scales, "scales", torch.float32)
    _dev(wpack, "wpack", torch.uint8)
    _dev(bias, "bias", torch.bfloat16)
    M, K = codes.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=codes.device)
    if workspace is None:
        workspace = alloc_workspace(256, codes.device)
    _check("hstu_gemm_e4m3", load_library().hstu_gemm_e4m3(
        _ptr(codes), _ptr(scales), ctypes.c_int64(M), ctypes.c_int32(K), _ptr(wpack), ctypes.c_int32(N),
        _ptr(bias), ctypes.c_int32(int(apply_silu)), _ptr(y), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
        _stream(stream)))
    return y


def hstu_jagged_truncate(seq_offsets, num_targets, keep: int, rows, *, out=None, out_offsets=None,
                         stream=None):
    """Attention truncation gather: each sequence's last min(hist, keep) history
    rows and all its candidates.  `rows` is any contiguous per-token tensor
    [T, ...] on the device.  Returns (out_offsets [B+1] int64, out) with `out`
    shaped like `rows` (T rows of room; the kept batch is out[:out_offsets[-1]])."""
    _dev(seq_offsets, "seq_offsets", torch.int64)
    _dev(num_targets, "num_targets", torch.int32)
    _dev(rows, "rows")
    B, T = seq_offsets.numel() - 1, rows.shape[0]
    row_bytes = rows.element_size() * math.prod(rows.shape[1:])
    if out is None:
        out = torch.empty_like(rows)
    if out_offsets is None:
        out_offsets = torch.empty(B + 1, dtype=torch.int64, device=rows.device)
    _dev(out, "out", rows.dtype)
    _dev(out_offsets, "out_offsets", torch.int64)
    _check("hstu_jagged_truncate", load_library().hstu_jagged_truncate(
        ctypes.c_int32(B), ctypes.c_int64(T), ctypes.c_int32(keep), _ptr(seq_offsets), _ptr(num_targets),
        _ptr(rows), ctypes.c_int64(row_bytes), _ptr(out), _ptr(out_offsets), _stream(stream)))
    return out_offsets, out


def hstu_check_device_flag(workspace: torch.Tensor, stream=None):
    """(status, bits) of the device input check of the last call on `workspace`."""
    bits = ctypes.c_int32(0)
    st = load_library().hstu_check_device_flag(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    return st, bits.value


def hstu_debug_bias_indices(desc: hstu_attn_desc, seq_offsets, timestamps, num_targets, rows,
                            stream=None):
    n = rows.shape[0]
    pos = torch.empty(n, dtype=torch.int32, device=rows.device)
    bkt = torch.empty(n, dtype=torch.int32, device=rows.device)
    _check("hstu_debug_bias_indices", load_library().hstu_debug_bias_indices(
        ctypes.byref(desc), _ptr(seq_offsets), _ptr(timestamps), _ptr(num_targets), _ptr(rows),
        ctypes.c_int64(n), _ptr(pos), _ptr(bkt), _stream(stream)))
    return pos, bkt


def hstu_debug_schedule(desc: hstu_attn_desc, seq_offsets, num_targets, is_bwd: bool,
                        tile_rows: int, stream=None):
    T, B = desc.total_tokens, desc.num_seqs
    cap = (T + tile_rows - 1) // tile_rows + B
    dev = seq_offsets.device
    items = torch.full((max(cap, 1), 2), -1, dtype=torch.int32, device=dev)
    count = torch.zeros(1, dtype=torch.int32, device=dev)
    hdr = torch.zeros(64, dtype=torch.int32, device=dev)
    _check("hstu_debug_schedule", load_library().hstu_debug_schedule(
        ctypes.byref(desc), _ptr(seq_offsets), _ptr(num_targets), int(is_bwd), int(tile_rows),
        _ptr(items), ctypes.c_int32(cap), _ptr(count), _ptr(hdr), _stream(stream)))
    return items, count, hdr
