"""B200 (sm_100a) Multi-head Latent Attention: absorbed decode over the latent cache.

A thin ctypes binding over the C ABI in include/mla.h (libmla_b200.so).  The functions
here only marshal arguments (torch tensors -> device pointers, the current CUDA stream);
every step of the computation runs in the library's CUDA kernels.  There is no fallback:
if the library is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python compressed_kv_cache_absorbed_b200/_build.py` (nvcc, sm_100a)")
_lib = ctypes.CDLL(LIB_PATH)

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE = 0, 1, 2, 3
MLA_ERR_CUDA, MLA_ERR_DEVICE_TIMEOUT, MLA_ERR_OUT_OF_RANGE, MLA_ERR_NO_MEMORY = 4, 5, 6, 7
MLA_F32, MLA_BF16 = 0, 1


class mla_dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_c", ctypes.c_int32),
                ("d_hR", ctypes.c_int32), ("qk_nope", ctypes.c_int32), ("v_head", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


_P = ctypes.c_void_p
_D = ctypes.POINTER(mla_dims)
_S = ctypes.c_int  # mla_status
SIGNATURES = {
    "mla_status_string": (ctypes.c_char_p, [_S]),
    "mla_last_cuda_error": (ctypes.c_char_p, []),
    "mla_cache_row_elems": (ctypes.c_int64, [_D]),
    "mla_cache_bytes_per_token": (ctypes.c_int64, [_D, ctypes.c_int32]),
    "mla_decode_path": (ctypes.c_int32, [_D]),
    "mla_absorb_weights": (_S, [_D, _P, _P, _P, _P, ctypes.c_int32, ctypes.POINTER(_P), _P]),
    "mla_weights_destroy": (_S, [_P]),
    "mla_append_cache": (_S, [_D, _P, _P, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_int64, _P]),
    "mla_decode_workspace_size": (ctypes.c_size_t, [_D, ctypes.c_int32]),
    "mla_decode_absorbed": (_S, [_D, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P, _P,
                                 ctypes.c_size_t, _P]),
    "mla_prefill_workspace_size": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int32]),
    "mla_prefill_causal": (_S, [_D, _P, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P,
                                ctypes.c_size_t, _P]),
    "mla_get_device_error": (_S, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "mla_decode_absorbed_noalloc": (_S, [_D, _P, _P, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P,
                                         _P]),
    "mla_decode_absorbed_paged": (_S, [_D, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P, ctypes.c_int32,
                                       _P, _P, ctypes.c_size_t, _P]),
    "mla_decode_absorbed_paged_multi": (_S, [_D, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P,
                                             ctypes.c_int32, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "mla_decode_multi_workspace_size": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]),
    "mla_decode_absorbed_host": (_S, [_D, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P, _P,
                                      ctypes.c_size_t, _P]),
    "mla_fp8_row_bytes": (ctypes.c_int64, [_D]),
    "mla_quantize_cache_fp8": (_S, [_D, _P, _P, ctypes.c_int32, _P, ctypes.c_int64, _P]),
    "mla_append_fp8_workspace_size": (ctypes.c_size_t, [_D, ctypes.c_int32]),
    "mla_append_cache_fp8": (_S, [_D, _P, _P, _P, _P, _P, ctypes.c_int32, _P, ctypes.c_int64, _P, ctypes.c_size_t,
                                  _P]),
    "mla_decode_absorbed_fp8": (_S, [_D, _P, _P, _P, _P, ctypes.c_int64, _P, ctypes.c_int32, _P, _P, ctypes.c_size_t,
                                     _P]),
    "mla_rope_apply": (_S, [_P, _P, ctypes.c_int64, _P, _P]),
    "mla_set_wait_limit": (_S, [ctypes.c_uint32]),
    "mla_test_starve_projection": (_S, [ctypes.c_int32]),
    "mla_profile_enable": (None, [ctypes.c_int32]),
    "mla_profile_report": (ctypes.c_int32, [ctypes.c_char_p, ctypes.c_size_t, ctypes.c_int32]),
}
for _name, (_res, _args) in SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class MLAError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.mla_status_string(status).decode()
        if status == MLA_ERR_CUDA:
            msg += f" ({_lib.mla_last_cuda_error().decode()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MLAError(status, where)


def make_dims(H, d_model, d_c, d_hR, qk_nope, v_head, dtype, softmax_scale=0.0,
              rope_theta=0.0) -> mla_dims:
    dt = {torch.float32: MLA_F32, torch.bfloat16: MLA_BF16, "f32": MLA_F32, "bf16": MLA_BF16}[dtype]
    return mla_dims(H, d_model, d_c, d_hR, qk_nope, v_head, softmax_scale, rope_theta, dt)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to the MLA library must be contiguous"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------- host helpers

def mla_cache_row_elems(dims: mla_dims) -> int:
    return int(_lib.mla_cache_row_elems(ctypes.byref(dims)))


def mla_cache_bytes_per_token(dims: mla_dims, layers: int = 1) -> int:
    return int(_lib.mla_cache_bytes_per_token(ctypes.byref(dims), layers))


def mla_decode_path(dims: mla_dims) -> int:
    return int(_lib.mla_decode_path(ctypes.byref(dims)))


def mla_decode_workspace_size(dims: mla_dims, B: int) -> int:
    return int(_lib.mla_decode_workspace_size(ctypes.byref(dims), B))


def mla_prefill_workspace_size(dims: mla_dims, B: int, S: int) -> int:
    return int(_lib.mla_prefill_workspace_size(ctypes.byref(dims), B, S))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A device byte buffer for a workspace (torch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# -------------------------------------------------------------------- weights

class MLAWeights:
    """Owner of an mla_weights handle (packed W_UK/W_UV; borrows W_Q/W_O; with fold, also the
    folded products)."""

    def __init__(self, dims: mla_dims, W_UK, W_UV, W_Q=None, W_O=None, stream=None, fold=False):
        self.dims = dims
        self._keep = (W_Q, W_O)  # borrowed by the handle: keep alive
        h = ctypes.c_void_p()
        _check(_lib.mla_absorb_weights(ctypes.byref(dims), _ptr(W_UK), _ptr(W_UV), _ptr(W_Q), _ptr(W_O),
                                       1 if fold else 0, ctypes.byref(h), _stream(stream)), "mla_absorb_weights")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _lib.mla_weights_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def mla_absorb_weights(dims, W_UK, W_UV, W_Q=None, W_O=None, stream=None, fold=False) -> MLAWeights:
    return MLAWeights(dims, W_UK, W_UV, W_Q, W_O, stream, fold)


# ------------------------------------------------------------------------ calls

def mla_append_cache(dims, h, W_DKV, W_KR, pos, slot, cache, stream=None) -> None:
    n = h.shape[0] if h.dim() == 2 else h.numel() // dims.d_model
    _check(_lib.mla_append_cache(ctypes.byref(dims), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(pos),
                                 _ptr(slot), n, _ptr(cache), cache.shape[0], _stream(stream)),
           "mla_append_cache")


def mla_decode_absorbed(dims, weights: MLAWeights, cache, offsets, out, ws, q_nope=None, q_rope=None,
                        h=None, q_pos=None, stream=None) -> None:
    B = offsets.numel() - 1
    _check(_lib.mla_decode_absorbed(ctypes.byref(dims), weights.handle, _ptr(q_nope), _ptr(q_rope),
                                    _ptr(h), _ptr(q_pos), _ptr(cache), cache.shape[0], _ptr(offsets), B,
                                    _ptr(out), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "mla_decode_absorbed")


def mla_decode_absorbed_noalloc(dims, weights: MLAWeights, cache, offsets, out, q_nope=None,
                                q_rope=None, h=None, q_pos=None, stream=None) -> None:
    """mla_decode_absorbed with the library's fixed device scratch instead of a workspace,
    for callers that cannot allocate device memory."""
    B = offsets.numel() - 1
    _check(_lib.mla_decode_absorbed_noalloc(ctypes.byref(dims), weights.handle, _ptr(q_nope), _ptr(q_rope),
                                            _ptr(h), _ptr(q_pos), _ptr(cache), cache.shape[0], _ptr(offsets), B,
                                            _ptr(out), _stream(stream)), "mla_decode_absorbed_noalloc")


def mla_decode_absorbed_paged(dims, weights: MLAWeights, cache_pages, block_table, seq_lens, out, ws, q_nope,
                              q_rope, stream=None) -> None:
    """Absorbed decode over a paged cache: cache_pages [num_pages, 64, d_c + d_hR],
    block_table int32 [B, max_blocks] (page of each 64-token block), seq_lens int32 [B]."""
    B, max_blocks = block_table.shape
    _check(_lib.mla_decode_absorbed_paged(ctypes.byref(dims), weights.handle, _ptr(q_nope), _ptr(q_rope),
                                          _ptr(cache_pages), cache_pages.shape[0], _ptr(block_table), max_blocks,
                                          _ptr(seq_lens), B, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "mla_decode_absorbed_paged")


def mla_decode_multi_workspace_size(dims, B: int, q_len: int, max_blocks: int) -> int:
    return _lib.mla_decode_multi_workspace_size(ctypes.byref(dims), B, q_len, max_blocks)


def mla_decode_absorbed_paged_multi(dims, weights: MLAWeights, cache_pages, block_table, seq_lens, out, ws,
                                    q_nope, q_rope, stream=None) -> None:
    """Multi-token decode over a paged cache: q_nope [B, q_len, H, qk_nope], q_rope
    [B, q_len, H, d_hR], out [B, q_len, H, v_head]; the q_len new tokens are the last
    q_len of each sequence's seq_lens[b] tokens (already appended to the pages)."""
    B, max_blocks = block_table.shape
    q_len = q_nope.shape[1]
    _check(_lib.mla_decode_absorbed_paged_multi(ctypes.byref(dims), weights.handle, _ptr(q_nope), _ptr(q_rope),
                                                _ptr(cache_pages), cache_pages.shape[0], _ptr(block_table),
                                                max_blocks, _ptr(seq_lens), B, q_len, _ptr(out), _ptr(ws),
                                                ws.numel(), _stream(stream)),
           "mla_decode_absorbed_paged_multi")


def mla_decode_absorbed_host(dims, weights: MLAWeights, cache, offsets, q_nope_host, q_rope_host, out_host, ws,
                             stream=None) -> None:
    """mla_decode_absorbed with q_nope, q_rope and the output in host (CPU, ideally pinned)
    tensors; the copies run on the stream inside the call.  Synchronise the stream before
    reading out_host."""
    B = offsets.numel() - 1
    _check(_lib.mla_decode_absorbed_host(ctypes.byref(dims), weights.handle, _ptr(q_nope_host), _ptr(q_rope_host),
                                         _ptr(cache), cache.shape[0], _ptr(offsets), B, _ptr(out_host), _ptr(ws),
                                         ws.numel(), _stream(stream)), "mla_decode_absorbed_host")


def mla_fp8_row_bytes(dims) -> int:
    """Bytes of one FP8 cache row (-1 for shapes without FP8 rows)."""
    return int(_lib.mla_fp8_row_bytes(ctypes.byref(dims)))


def mla_quantize_cache_fp8(dims, rows, cache_fp8, slot=None, stream=None) -> None:
    """FP8 rows of bf16 cache rows [n, d_c + d_hR] into cache_fp8 (uint8 [capacity, row bytes])
    at slot (int64 [n], device) or at rows 0 .. n-1."""
    _check(_lib.mla_quantize_cache_fp8(ctypes.byref(dims), _ptr(rows), _ptr(slot), rows.shape[0], _ptr(cache_fp8),
                                       cache_fp8.shape[0], _stream(stream)), "mla_quantize_cache_fp8")


def mla_append_fp8_workspace_size(dims, n: int) -> int:
    return int(_lib.mla_append_fp8_workspace_size(ctypes.byref(dims), n))


def mla_append_cache_fp8(dims, h, W_DKV, W_KR, pos, slot, cache_fp8, ws, stream=None) -> None:
    """mla_append_cache into an FP8 cache (uint8 [capacity, row bytes])."""
    n = h.shape[0]
    _check(_lib.mla_append_cache_fp8(ctypes.byref(dims), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(pos), _ptr(slot), n,
                                     _ptr(cache_fp8), cache_fp8.shape[0], _ptr(ws), ws.numel(), _stream(stream)),
           "mla_append_cache_fp8")


def mla_decode_absorbed_fp8(dims, weights: MLAWeights, cache_fp8, offsets, out, ws, q_nope, q_rope,
                            stream=None) -> None:
    """mla_decode_absorbed over an FP8 cache (uint8 [rows, row bytes])."""
    B = offsets.numel() - 1
    _check(_lib.mla_decode_absorbed_fp8(ctypes.byref(dims), weights.handle, _ptr(q_nope), _ptr(q_rope),
                                        _ptr(cache_fp8), cache_fp8.shape[0], _ptr(offsets), B, _ptr(out), _ptr(ws),
                                        ws.numel(), _stream(stream)), "mla_decode_absorbed_fp8")


def mla_prefill_causal(dims, weights: MLAWeights, h, W_DKV, W_KR, cache, out, ws, stream=None) -> None:
    B, S = h.shape[0], h.shape[1]
    _check(_lib.mla_prefill_causal(ctypes.byref(dims), weights.handle, _ptr(h), _ptr(W_DKV), _ptr(W_KR),
                                   _ptr(cache), _ptr(out), B, S, _ptr(ws), ws.numel(), _stream(stream)),
           "mla_prefill_causal")


def mla_get_device_error(stream=None):
    """(status, detail) of the device error word (synchronises the stream, then clears it)."""
    d = ctypes.c_int64(0)
    st = _lib.mla_get_device_error(_stream(stream), ctypes.byref(d))
    return int(st), int(d.value)


def mla_rope_apply(x, cos_sin, y, stream=None) -> None:
    """y = the RoPE pairs of x (float32 [..., 2k]) rotated by cos_sin (float64 [..., k, 2])."""
    _check(_lib.mla_rope_apply(_ptr(x), _ptr(cos_sin), x.numel() // 2, _ptr(y), _stream(stream)), "mla_rope_apply")


def mla_set_wait_limit(polls: int) -> None:
    """Polls each bounded device wait makes before giving up (0 = the default); a test hook."""
    _check(_lib.mla_set_wait_limit(int(polls)), "mla_set_wait_limit")


def mla_test_starve_projection(on: bool) -> None:
    """While on, the projection GEMM's loader issues no loads so its waits run out (test hook)."""
    _check(_lib.mla_test_starve_projection(1 if on else 0), "mla_test_starve_projection")


def mla_profile_enable(on: bool = True) -> None:
    _lib.mla_profile_enable(1 if on else 0)


def mla_profile_report(reset: bool = True) -> dict:
    """{kernel_name: (launches, total_ms)} of the library's own launches since the last reset."""
    buf = ctypes.create_string_buffer(1 << 16)
    _lib.mla_profile_report(buf, len(buf), 1 if reset else 0)
    out = {}
    for line in buf.value.decode().splitlines():
        name, n, ms = line.split()
        out[name] = (int(n), float(ms))
    return out


def lib():
    return _lib
