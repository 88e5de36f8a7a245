"""Tolerances and small utilities shared by the parity tests.

Tolerances (written once, used everywhere):
  fp32 storage:  |x - y| <= 1e-5 |y| + 1e-5 RMS(y), elementwise
  bf16 storage:  max |x - y| <= 2e-2 RMS(y)
  RMS(y) is taken per output vector: one head's v_head outputs for one query, or one
  token's d_model outputs after W_O (a t = 0 prefill row is ~N(0,1) while late rows are
  averages ~10x smaller, so one RMS over all rows would sit below the bf16 rounding of the
  large rows).
  cache values:  bf16 rows: layout bit-exact (only the addressed rows change, c then k_rope);
                 each value within 1 bf16 ulp of the oracle's nearest-even rounding, or within
                 2^-16 RMS absolute (fp32 accumulation error of a d_model-long dot product,
                 ~sqrt(K) 2^-24 RMS, can exceed one ulp of a near-zero value); at least 99% of
                 values bit-exact.  fp32 rows within the fp32 tolerance above
where y is the float64 oracle and x the CUDA result.
"""
from __future__ import annotations

import numpy as np
import torch

FP32_REL = 1e-5
BF16_RMS = 2e-2
CACHE_ABS_RMS = 2.0 ** -16
CACHE_EXACT_FRAC = 0.99


def np64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def rms(y) -> float:
    y = np64(y)
    return float(np.sqrt(np.mean(y * y))) if y.size else 0.0


# (what, dtype, worst err/limit) of every comparison made in this process; the session summary
# prints the closest ones (conftest.py)
RATIOS: list = []


def assert_close(x, y, dtype: str, what: str = "") -> dict:
    """Compare per output vector (the last axis: one head's v_head values, or one token's
    d_model values); the RMS in each tolerance is that vector's RMS."""
    x, y = np64(x), np64(y)
    assert x.shape == y.shape, f"{what}: shape {x.shape} vs {y.shape}"
    assert np.all(np.isfinite(x)), f"{what}: non-finite values in the CUDA result"
    if x.size == 0:
        return {"max_err": 0.0, "worst_ratio": 0.0}
    x2, y2 = x.reshape(-1, x.shape[-1]), y.reshape(-1, y.shape[-1])
    err = np.abs(x2 - y2)
    r = np.sqrt(np.mean(y2 * y2, axis=1, keepdims=True))
    if dtype == "f32":
        lim = FP32_REL * np.abs(y2) + FP32_REL * r
    else:
        lim = np.broadcast_to(BF16_RMS * r, err.shape)
    bad = err > lim
    worst = float(np.max(err / np.maximum(lim, 1e-300)))
    RATIOS.append((what, dtype, worst))
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {err.size} elements over the {dtype} tolerance; "
                           f"worst err/limit {worst:.3f}, max err {err.max():.3e}")
    return {"max_err": float(err.max()), "worst_ratio": worst}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between bf16 bit patterns (same sign assumed
    for nonzero neighbours; sign-magnitude mapped to a monotone integer line)."""
    def line(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(line(a_bits) - line(b_bits))


def to_dev(d: dict, device="cuda") -> dict:
    return {k: v.to(device) for k, v in d.items()}
