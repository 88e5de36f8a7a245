"""float64 CPU oracle for MLA (naive, with K and V materialised; plus the absorbed form).

TEST INFRASTRUCTURE.  Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  It shares no code with the CUDA library; the two meet
only through the seeded inputs of `workloads`.

The arithmetic lives in `mla_oracle.c` (plain C, one loop per sum, float64).  This module
converts inputs to contiguous float64 arrays and calls it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

from . import build as _build

_lib = None
_I32 = ctypes.c_int
_I64 = ctypes.c_int64
_D = ctypes.c_double
_P = ctypes.c_void_p


def load(path: Optional[str] = None):
    """Load (building it first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    if _lib is None:
        if not os.path.exists(_build.LIB) or os.path.getmtime(_build.LIB) < os.path.getmtime(_build.SRC):
            _build.build()
        _lib = _declare(ctypes.CDLL(_build.LIB))
    return _lib


def _declare(lib):
    lib.oracle_mha_elems_per_token.restype = _I64
    lib.oracle_mha_elems_per_token.argtypes = [_I64, _I64]
    lib.oracle_mla_elems_per_token.restype = _I64
    lib.oracle_mla_elems_per_token.argtypes = [_I64, _I64, _I64]
    lib.oracle_round_bf16.restype = ctypes.c_uint16
    lib.oracle_round_bf16.argtypes = [_D]
    lib.oracle_round_bf16_array.argtypes = [_I64, _P, _P]
    lib.oracle_round_e4m3.restype = _D
    lib.oracle_round_e4m3.argtypes = [_D]
    lib.oracle_quantize_latent_fp8.argtypes = [_I32, _I32, _I32, _P, _P, _P]
    lib.oracle_e4m3_bits.restype = ctypes.c_uint8
    lib.oracle_e4m3_bits.argtypes = [_D]
    lib.oracle_fp8_row_f32.argtypes = [_I32, _I32, _P, _I32, _P, _P]
    lib.oracle_rope.argtypes = [_I32, _P, _D, _D, _P]
    lib.oracle_rope_pairs_f32.argtypes = [_I64, _P, _P, _P]
    lib.oracle_latent_rows.argtypes = [_I32, _I32, _I32, _I32, _P, _P, _P, _P, _D, _P]
    lib.oracle_query.argtypes = [_I32, _I32, _I32, _I32, _I32, _P, _P, _P, _D, _P, _P]
    att = [_I32, _I32, _I32, _I32, _I32, _D, _P, _P, _P, _P, _P, _P, _P, _P]
    lib.oracle_attend_naive.argtypes = att
    lib.oracle_attend_absorbed.argtypes = att
    lib.oracle_attend_probs.argtypes = att[:-1]
    lib.oracle_decode.argtypes = [_I32, _I32, _I32, _I32, _I32, _I32, _D, _P, _P, _P, _P, _P, _P,
                                  _I32, _P, _P, _P, _P]
    lib.oracle_decode_multi.argtypes = [_I32, _I32, _I32, _I32, _I32, _I32, _I32, _D, _P, _P, _P, _P, _P,
                                        _P, _I32, _P, _P, _P, _P]
    lib.oracle_out_proj.argtypes = [_I32, _I32, _I32, _P, _P, _P]
    lib.oracle_prefill_head.argtypes = [_I32, _I32, _I32, _I32, _I32, _I32, _D, _P, _P, _P, _P, _P,
                                        _I32, _P, _P]
    return lib


def f64(x) -> np.ndarray:
    """Any tensor/array (float32, bfloat16, float64) as a contiguous float64 numpy array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x), dtype=np.int32)


def _i64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x), dtype=np.int64)


# --------------------------------------------------------------------------- sizes

def mha_elems_per_token(n_heads: int, d_head: int, lib=None) -> int:
    return int((lib or load()).oracle_mha_elems_per_token(n_heads, d_head))


def mla_elems_per_token(d_c: int, d_hR: int, layers: int = 1, lib=None) -> int:
    return int((lib or load()).oracle_mla_elems_per_token(d_c, d_hR, layers))


# ------------------------------------------------------------------------ rounding

def round_bf16(x, lib=None) -> np.ndarray:
    """float64 -> bfloat16 bit patterns (uint16), one rounding, nearest-even."""
    a = f64(x)
    out = np.empty(a.shape, dtype=np.uint16)
    (lib or load()).oracle_round_bf16_array(a.size, _p(a), _p(out))
    return out


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------- RoPE

def round_e4m3(x, lib=None) -> np.ndarray:
    """Nearest FP8 E4M3 value (ties to even, saturating at 448) of each element, as float64."""
    x = f64(x)
    fn = (lib or load()).oracle_round_e4m3
    return np.array([fn(float(v)) for v in x.reshape(-1)]).reshape(x.shape)


def quantize_latent_fp8(rows, d_c: int, lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """Per-token FP8 E4M3 latent: (dequantised rows [n, d_c + d_hR], scales [n])."""
    rows = f64(rows)
    n, rw = rows.shape
    deq = np.empty_like(rows)
    scales = np.empty(n)
    (lib or load()).oracle_quantize_latent_fp8(n, d_c, rw - d_c, _p(rows), _p(deq), _p(scales))
    return deq, scales


def e4m3_bits(x, lib=None) -> np.ndarray:
    """The E4M3 byte of each value (values as round_e4m3 returns them)."""
    x = f64(x)
    fn = (lib or load()).oracle_e4m3_bits
    return np.array([fn(float(v)) for v in x.reshape(-1)], dtype=np.uint8).reshape(x.shape)


def fp8_rows_f32(rows, d_c: int, row_bytes: int, lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """FP8 cache rows of bf16-valued rows [n, d_c + d_hR], every decision in float:
    (bytes uint8 [n, row_bytes], dequantised rows float64 [n, d_c + d_hR])."""
    rows = f64(rows)
    n, rw = rows.shape
    out = np.zeros((n, row_bytes), dtype=np.uint8)
    deq = np.empty_like(rows)
    fn = (lib or load()).oracle_fp8_row_f32
    for i in range(n):
        fn(d_c, rw - d_c, _p(rows[i]), row_bytes, _p(out[i]), _p(deq[i]))
    return out, deq


def rope_pairs_f32(x, cos_sin, lib=None) -> np.ndarray:
    """float32 pairs rotated by given (cos, sin) in double, each operation rounded, then
    rounded to float32 (the kernels' rotation arithmetic)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    cs = np.ascontiguousarray(np.asarray(cos_sin, dtype=np.float64))
    assert cs.size == x.size
    y = np.empty_like(x)
    (lib or load()).oracle_rope_pairs_f32(x.size // 2, _p(x), _p(cs), _p(y))
    return y


def rope(x, pos: float, theta: float = 10000.0, lib=None) -> np.ndarray:
    a = f64(x)
    out = np.empty_like(a)
    (lib or load()).oracle_rope(a.shape[-1], _p(a), float(pos), float(theta), _p(out))
    return out


# ----------------------------------------------------------------- cache / query

def latent_rows(h, W_DKV, W_KR, pos, theta: float = 10000.0, lib=None) -> np.ndarray:
    """Cache rows [n, d_c + d_hR] = [W_DKV h | RoPE(W_KR h, pos)] in float64."""
    h, W_DKV, W_KR = f64(h), f64(W_DKV), f64(W_KR)
    n, d_model = h.shape
    d_c, d_hR = W_DKV.shape[0], W_KR.shape[0]
    pos = _i32(pos)
    rows = np.empty((n, d_c + d_hR))
    (lib or load()).oracle_latent_rows(n, d_model, d_c, d_hR, _p(h), _p(W_DKV), _p(W_KR), _p(pos),
                                       float(theta), _p(rows))
    return rows


def query(h, W_Q, pos, H: int, qk_nope: int, d_hR: int, theta: float = 10000.0,
          lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """(q_nope [n,H,qk_nope], q_rope [n,H,d_hR]) from q = W_Q h with RoPE on the rotary part."""
    h, W_Q = f64(h), f64(W_Q)
    n, d_model = h.shape
    pos = _i32(pos)
    qn = np.empty((n, H, qk_nope))
    qr = np.empty((n, H, d_hR))
    (lib or load()).oracle_query(n, d_model, H, qk_nope, d_hR, _p(h), _p(W_Q), _p(pos), float(theta),
                                 _p(qn), _p(qr))
    return qn, qr


# -------------------------------------------------------------------------- decode

def attend(q_nope, q_rope, rows, W_UK_h, W_UV_h, scale: float, absorbed: bool = False,
           lib=None) -> Tuple[np.ndarray, np.ndarray, float]:
    """One head, one query over T rows -> (o [v_head], p [T], lse)."""
    qn, qr, rows, wk, wv = f64(q_nope), f64(q_rope), f64(rows), f64(W_UK_h), f64(W_UV_h)
    T = rows.shape[0]
    qk_nope, d_c = wk.shape
    v_head = wv.shape[0]
    d_hR = qr.shape[0]
    o = np.empty(v_head)
    p = np.empty(max(T, 1))
    lse = np.empty(1)
    fn = (lib or load()).oracle_attend_absorbed if absorbed else (lib or load()).oracle_attend_naive
    fn(T, d_c, d_hR, qk_nope, v_head, float(scale), _p(qn), _p(qr), _p(rows), _p(wk), _p(wv), _p(o),
       _p(p), _p(lse))
    return o, p[:T], float(lse[0])


def decode(q_nope, q_rope, rows, offsets, W_UK, W_UV, scale: float,
           units: Optional[Sequence[Tuple[int, int]]] = None, absorbed: bool = False,
           lib=None) -> Tuple[np.ndarray, np.ndarray]:
    """Decode attention per (b, h) unit.

    rows: [total, d_c+d_hR]; offsets: [B+1]; q_nope [B,H,qk_nope]; q_rope [B,H,d_hR].
    Returns (o, lse): o is [B,H,v_head] when units is None, else [len(units), v_head].
    """
    qn, qr, rows, wk, wv = f64(q_nope), f64(q_rope), f64(rows), f64(W_UK), f64(W_UV)
    B, H, qk_nope = qn.shape
    d_hR = qr.shape[2]
    d_c = wk.shape[2]
    v_head = wv.shape[1]
    offs = _i64(offsets)
    if units is None:
        ub = np.repeat(np.arange(B), H).astype(np.int32)
        uh = np.tile(np.arange(H), B).astype(np.int32)
    else:
        ub = _i32([u[0] for u in units])
        uh = _i32([u[1] for u in units])
    n = len(ub)
    o = np.empty((n, v_head))
    lse = np.empty(n)
    (lib or load()).oracle_decode(int(absorbed), H, d_c, d_hR, qk_nope, v_head, float(scale), _p(offs),
                                  _p(qn), _p(qr), _p(rows), _p(wk), _p(wv), n, _p(ub), _p(uh), _p(o),
                                  _p(lse))
    if units is None:
        return o.reshape(B, H, v_head), lse.reshape(B, H)
    return o, lse


def decode_multi(q_nope, q_rope, rows, offsets, W_UK, W_UV, scale: float,
                 units: Optional[Sequence[Tuple[int, int, int]]] = None, absorbed: bool = False,
                 lib=None) -> np.ndarray:
    """Multi-token decode per (b, t, h) unit: new token t of sequence b (the last q_len rows
    of the sequence are the new tokens) attends to the sequence's rows up to its own.

    rows: [total, d_c+d_hR]; offsets: [B+1]; q_nope [B,q_len,H,qk_nope]; q_rope [B,q_len,H,d_hR].
    Returns o: [B,q_len,H,v_head] when units is None, else [len(units), v_head].
    """
    qn, qr, rows, wk, wv = f64(q_nope), f64(q_rope), f64(rows), f64(W_UK), f64(W_UV)
    B, q_len, H, qk_nope = qn.shape
    d_hR = qr.shape[3]
    d_c = wk.shape[2]
    v_head = wv.shape[1]
    offs = _i64(offsets)
    if units is None:
        units = [(b, t, h) for b in range(B) for t in range(q_len) for h in range(H)]
    ub = _i32([u[0] for u in units])
    ut = _i32([u[1] for u in units])
    uh = _i32([u[2] for u in units])
    n = len(ub)
    o = np.empty((n, v_head))
    (lib or load()).oracle_decode_multi(int(absorbed), H, q_len, d_c, d_hR, qk_nope, v_head, float(scale),
                                        _p(offs), _p(qn), _p(qr), _p(rows), _p(wk), _p(wv), n, _p(ub), _p(ut),
                                        _p(uh), _p(o))
    if n == B * q_len * H and list(units) == [(b, t, h) for b in range(B) for t in range(q_len)
                                              for h in range(H)]:
        return o.reshape(B, q_len, H, v_head)
    return o


def out_proj(o, W_O, lib=None) -> np.ndarray:
    """out [n, d_model] = W_O concat_h o[n, h, :]."""
    o = f64(o)
    n = o.shape[0]
    o = o.reshape(n, -1)
    W_O = f64(W_O)
    d_model, Hv = W_O.shape
    out = np.empty((n, d_model))
    (lib or load()).oracle_out_proj(n, Hv, d_model, _p(o), _p(W_O), _p(out))
    return out


def prefill_head(q_nope, q_rope, rows, W_UK_h, W_UV_h, scale: float, t_list,
                 absorbed: bool = False, lib=None) -> np.ndarray:
    """Causal attention of one head of one sequence for query positions t_list -> [n_t, v_head].

    q_nope [S, qk_nope], q_rope [S, d_hR] (rotated), rows [S, d_c+d_hR]."""
    qn, qr, rows, wk, wv = f64(q_nope), f64(q_rope), f64(rows), f64(W_UK_h), f64(W_UV_h)
    S = rows.shape[0]
    qk_nope, d_c = wk.shape
    v_head = wv.shape[0]
    d_hR = qr.shape[1]
    tl = _i32(t_list)
    o = np.empty((len(tl), v_head))
    (lib or load()).oracle_prefill_head(int(absorbed), S, d_c, d_hR, qk_nope, v_head, float(scale),
                                        _p(qn), _p(qr), _p(rows), _p(wk), _p(wv), len(tl), _p(tl),
                                        _p(o))
    return o
