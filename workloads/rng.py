"""Seeded, counter-based synthetic inputs shared by the oracle side and the CUDA side.

This module draws numbers and rounds them to a storage type; it holds none of the
attention arithmetic.  Every value is a pure function of (seed, tensor_id, index):

* splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014): state_n = key + n * 0x9E3779B97F4A7C15, output = mix64(state_n) with the
  published finaliser constants.  The stream key is mix64(mix64(seed) ^ tensor_id * C).
* uniform double in (0, 1): ((u >> 11) + 0.5) * 2**-53.
* N(0, 1): Box-Muller, cosine branch only, using counters 2i and 2i+1 for sample i.
* integers in [lo, hi]: Lemire's multiply-shift on the high 32 bits (no rejection step;
  the bias is below 2**-15 for the ranges used here).
* bf16: float64 -> float32 (round to nearest even) -> bfloat16 (round to nearest even),
  done on the bit pattern.

numpy uint64 arithmetic wraps modulo 2**64, which is exactly what splitmix64 needs.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TID = np.uint64(0xD1B54A32D192ED03)
_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = _mix64(np.array([seed], dtype=np.uint64))[0]
        return _mix64(np.array([s ^ (np.uint64(tensor_id) * _TID)], dtype=np.uint64))[0]


def _u64(key: np.uint64, start: int, count: int) -> np.ndarray:
    with np.errstate(over="ignore"):
        n = np.arange(start + 1, start + 1 + count, dtype=np.uint64)
        return _mix64(key + n * GOLDEN)


def _uniform01(u: np.ndarray) -> np.ndarray:
    return ((u >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, tensor_id: int, n: int, std: float = 1.0, store: str = "f64") -> np.ndarray:
    """n samples of N(0, std**2), stored as float64 ("f64"), float32 ("f32", round to
    nearest even) or bfloat16 bit patterns ("bf16", uint16)."""
    key = stream_key(seed, tensor_id)
    out = np.empty(n, dtype={"f64": np.float64, "f32": np.float32, "bf16": np.uint16}[store])

    def fill(s: int) -> None:
        m = min(_CHUNK, n - s)
        u = _u64(key, 2 * s, 2 * m)
        u1 = _uniform01(u[0::2])
        u2 = _uniform01(u[1::2])
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2) * std
        if store == "bf16":
            out[s:s + m] = f64_to_bf16_bits(z)
        else:
            out[s:s + m] = z

    starts = range(0, n, _CHUNK)
    if n <= _CHUNK:
        for s in starts:
            fill(s)
    else:
        # chunks are independent (counter-based), so the result does not depend on threading
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    return out


def randint(seed: int, tensor_id: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n integers in [lo, hi] inclusive as int64."""
    key = stream_key(seed, tensor_id)
    u = _u64(key, 0, n)
    span = np.uint64(hi - lo + 1)
    with np.errstate(over="ignore"):
        r = ((u >> np.uint64(32)) * span) >> np.uint64(32)
    return r.astype(np.int64) + lo


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 -> float32 -> bfloat16 (both round to nearest even); returns uint16 bits."""
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
