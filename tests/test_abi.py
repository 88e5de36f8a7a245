"""The C-ABI library loads, exports every declared symbol, and its host-only logic is right
(no GPU needed: nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest

import oracle
import compressed_kv_cache_absorbed_b200 as mla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ("mla_absorb_weights", "mla_append_cache", "mla_decode_absorbed", "mla_prefill_causal"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mla.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    assert set(declared_functions()) <= set(mla.SIGNATURES)


def v3(dtype="bf16", **kw):
    d = dict(H=128, d_model=7168, d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype=dtype)
    d.update(kw)
    return mla.make_dims(**d)


def test_cache_row_matches_the_oracle_and_the_pages():
    # (d_c + d_hR) elements per token per layer: 576 for V2/V3; 35136 over V3's 61 layers
    d = v3()
    assert mla.mla_cache_row_elems(d) == oracle.mla_elems_per_token(512, 64, 1) == 576
    assert mla.mla_cache_bytes_per_token(d, 61) == 35136 * 2
    assert mla.mla_cache_bytes_per_token(v3("f32"), 1) == 576 * 4
    assert mla.mla_cache_row_elems(v3(H=0)) == -1


def test_decode_path_selection():
    assert mla.mla_decode_path(v3()) == 1                     # bf16 V2/V3 head shape: tcgen05
    assert mla.mla_decode_path(v3(dtype="f32")) == 0
    assert mla.mla_decode_path(v3(d_hR=63)) == -1              # odd rotary width
    assert mla.mla_decode_path(v3(d_c=1024)) == -1             # wider than the kernels
    tiny = mla.make_dims(4, 256, 64, 16, 32, 32, "f32")
    assert mla.mla_decode_path(tiny) == 0


def test_workspace_sizes_are_positive_and_monotone():
    d = v3()
    a, b = mla.mla_decode_workspace_size(d, 8), mla.mla_decode_workspace_size(d, 64)
    assert 0 < a < b
    assert mla.mla_decode_workspace_size(v3(H=0), 8) == 0
    # multi-token decode: the decode workspace of B * q_len sequences plus the per-token
    # block table; invalid sizes give 0
    m1, m4 = mla.mla_decode_multi_workspace_size(d, 8, 1, 64), mla.mla_decode_multi_workspace_size(d, 8, 4, 64)
    assert mla.mla_decode_workspace_size(d, 8) < m1 < m4
    assert m4 >= mla.mla_decode_workspace_size(d, 32) + 32 * 64 * 4
    assert mla.mla_decode_multi_workspace_size(d, 8, 0, 64) == 0
    assert mla.mla_decode_multi_workspace_size(d, 8, 2, 0) == 0
    assert mla.mla_decode_multi_workspace_size(d, 1 << 20, 1 << 12, 64) == 0
    assert mla.mla_decode_multi_workspace_size(v3(H=64), 8, 2, 64) == 0   # tensor-core shape only
    p = mla.mla_prefill_workspace_size(v3(d_model=5120), 4, 4096)
    # q (192) + K_nope (128) + V (128) per token and head, bf16
    assert p >= 4 * 4096 * 128 * (192 + 128 + 128) * 2


def test_status_strings():
    for s in range(8):
        assert mla.lib().mla_status_string(s).decode().startswith("MLA_")


def test_argument_errors_return_before_any_launch():
    d = v3()
    lib = mla.lib()
    # negative counts, missing pointers and bad dims are rejected on the host
    assert lib.mla_append_cache(ctypes.byref(d), None, None, None, None, None, -1, None, 0, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_append_cache(ctypes.byref(d), None, None, None, None, None, 0, None, 0, None) == mla.MLA_OK
    assert lib.mla_append_cache(ctypes.byref(d), None, None, None, None, None, 4, None, 10, None) == mla.MLA_ERR_INVALID_ARG
    bad = v3(d_hR=7)
    assert lib.mla_append_cache(ctypes.byref(bad), None, None, None, None, None, 1, None, 1, None) == mla.MLA_ERR_UNSUPPORTED
    h = ctypes.c_void_p()
    assert lib.mla_absorb_weights(ctypes.byref(d), None, None, None, None, 0, ctypes.byref(h), None) == mla.MLA_ERR_INVALID_ARG
    # fold needs W_Q and W_O; fold outside {0, 1} is rejected (both before any device work)
    dummy = ctypes.c_void_p(16)
    assert lib.mla_absorb_weights(ctypes.byref(d), dummy, dummy, None, None, 1, ctypes.byref(h), None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_weights(ctypes.byref(d), dummy, dummy, None, None, 2, ctypes.byref(h), None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_absorbed(ctypes.byref(d), None, None, None, None, None, None, 0, None, 1, None, None, 0, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_prefill_causal(ctypes.byref(d), None, None, None, None, None, None, 1, 1, None, 0, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_absorbed_paged(ctypes.byref(d), None, None, None, None, 1, None, 1, None, 1, None, None,
                                         0, None) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_absorbed_host(ctypes.byref(d), None, None, None, None, 1, None, 1, None, None, 0,
                                        None) == mla.MLA_ERR_INVALID_ARG
    multi = lambda B, q_len: lib.mla_decode_absorbed_paged_multi(ctypes.byref(d), None, None, None, None, 1, None,
                                                                 1, None, B, q_len, None, None, 0, None)
    assert multi(1, 2) == mla.MLA_ERR_INVALID_ARG      # no weights handle
    assert multi(1, 0) == mla.MLA_ERR_INVALID_ARG      # q_len < 1
    assert multi(-1, 2) == mla.MLA_ERR_INVALID_ARG
    assert lib.mla_weights_destroy(None) == mla.MLA_OK
