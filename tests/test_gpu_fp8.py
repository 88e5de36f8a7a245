"""The FP8 latent cache on a B200, through the C ABI: the quantisation kernel against the
oracle's float-decision rows byte for byte, the append into FP8 rows, and the FP8 decode
against the float64 oracle decode on the oracle's dequantised rows."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import assert_close, np64

pytestmark = pytest.mark.gpu

mla = pytest.importorskip("compressed_kv_cache_absorbed_b200")

DEV = "cuda"
V3 = workloads.WORKLOADS["v3_decode_b32_ctx4096"]


def dims_v3(d_model=0):
    return mla.make_dims(128, d_model, 512, 64, 128, 128, "bf16")


def bf16_rows(n, seed, scale=0.5):
    r = np.random.default_rng(seed)
    x = r.standard_normal((n, 576)) * scale
    return torch.from_numpy(x).to(torch.bfloat16)


def test_quantised_rows_are_the_oracles_bytes():
    """Codes, rotary bytes, scale and padding of every row equal the oracle's float-decision
    row; rows not addressed keep their sentinel bytes; a slot outside the cache latches."""
    dims = dims_v3()
    nb = mla.mla_fp8_row_bytes(dims)
    assert nb == 656
    rows = bf16_rows(300, 71)
    rows[5, :512] = 0                                       # zero latent: scale 1, codes 0
    rows[6, :512] *= 300                                    # large values
    rows[7, :512] *= 1e-6                                   # tiny values (subnormal codes)
    rows[8, 3] = -0.0
    n, cap = rows.shape[0], 333
    slots = np.random.default_rng(72).choice(cap, n, replace=False).astype(np.int64)
    cache = torch.full((cap, nb), 0xA5, dtype=torch.uint8, device=DEV)
    mla.mla_quantize_cache_fp8(dims, rows.to(DEV), cache, slot=torch.from_numpy(slots).to(DEV))
    assert mla.mla_get_device_error() == (0, 0)
    want, _ = oracle.fp8_rows_f32(rows, 512, nb)
    got = cache.cpu().numpy()
    assert np.array_equal(got[slots], want), f"{int((got[slots] != want).sum())} bytes differ"
    rest = np.setdiff1d(np.arange(cap), slots)
    assert np.all(got[rest] == 0xA5)
    bad = torch.tensor([0, cap, -1], dtype=torch.int64, device=DEV)
    mla.mla_quantize_cache_fp8(dims, rows[:3].to(DEV), cache, slot=bad)
    st, _ = mla.mla_get_device_error()
    assert st == mla.MLA_ERR_OUT_OF_RANGE


def test_append_into_fp8_rows():
    """The append path (down-projection, RoPE, quantisation) for V3-sized tokens: at least
    99% of the codes are the oracle's (its bf16 rows, float decisions), the rest one E4M3
    step away (the fp32 accumulation can move a bf16 row value by an ulp); other rows are
    untouched."""
    w = workloads.WORKLOADS["v3_layer_b128_ctx8192"]
    d = workloads.make_weights(w)
    dims = mla.make_dims(w.H, w.d_model, w.d_c, w.d_hR, w.qk_nope, w.v_head, "bf16")
    n = 64
    h = torch.from_numpy(np.random.default_rng(73).standard_normal((n, w.d_model))).to(torch.bfloat16)
    pos = np.random.default_rng(74).integers(0, 40000, n).astype(np.int32)
    cap = 200
    slots = np.random.default_rng(75).choice(cap, n, replace=False).astype(np.int64)
    nb = mla.mla_fp8_row_bytes(dims)
    cache = torch.zeros((cap, nb), dtype=torch.uint8, device=DEV)
    ws = mla.workspace(mla.mla_append_fp8_workspace_size(dims, n))
    mla.mla_append_cache_fp8(dims, h.to(DEV), d["W_DKV"].to(DEV), d["W_KR"].to(DEV), torch.from_numpy(pos).to(DEV),
                             torch.from_numpy(slots).to(DEV), cache, ws)
    assert mla.mla_get_device_error() == (0, 0)
    rows64 = oracle.latent_rows(h, d["W_DKV"], d["W_KR"], pos, w.rope_theta)
    rows_bf = oracle.bf16_value(oracle.round_bf16(rows64))
    want, deq = oracle.fp8_rows_f32(rows_bf, 512, nb)
    got = cache.cpu().numpy()[slots]
    codes_g = torch.from_numpy(got[:, :512].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    codes_w = torch.from_numpy(want[:, :512].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    exact = (got[:, :512] == want[:, :512]).mean()
    assert exact >= 0.99, f"only {exact:.4f} of the codes are the oracle's"
    s_g = got[:, 640:644].copy().view(np.float32)[:, 0].astype(np.float64)
    s_w = want[:, 640:644].copy().view(np.float32)[:, 0].astype(np.float64)
    assert np.all(np.abs(s_g - s_w) <= 2.0 ** -7 * s_w), "scales within a bf16 ulp of the row maximum"
    # every dequantised value within one E4M3 step (2^-3 relative, 2^-9 subnormal) of the oracle's
    dq_g, dq_w = codes_g * s_g[:, None], codes_w * s_w[:, None]
    assert np.all(np.abs(dq_g - dq_w) <= 2.0 ** -3 * np.abs(dq_w) + 2.0 ** -8 * s_w[:, None])
    assert not cache.cpu().numpy()[np.setdiff1d(np.arange(cap), slots)].any()


def fp8_inputs(lengths, seed):
    w = workloads.shrink(V3, B=len(lengths), seed=seed)
    d = workloads.make_weights(w)
    r = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    rows = (torch.from_numpy(r.standard_normal((int(offs[-1]), w.row))) * 0.5).to(torch.bfloat16)
    d["offsets"] = torch.from_numpy(offs)
    d["rows"] = rows
    d["q_nope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.qk_nope))).to(torch.bfloat16)
    d["q_rope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.d_hR))).to(torch.bfloat16)
    return w, d


def run_fp8_decode(w, inp, rows_dev_fp8):
    dims = dims_v3()
    B = inp["offsets"].numel() - 1
    weights = mla.mla_absorb_weights(dims, inp["W_UK"].to(DEV), inp["W_UV"].to(DEV))
    out = torch.empty(B, w.H, w.v_head, dtype=torch.bfloat16, device=DEV)
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, B))
    mla.mla_decode_absorbed_fp8(dims, weights, rows_dev_fp8, inp["offsets"].to(DEV), out, ws,
                                inp["q_nope"].to(DEV), inp["q_rope"].to(DEV))
    assert mla.mla_get_device_error() == (0, 0)
    weights.close()
    return out.cpu()


def oracle_fp8_units(w, inp, deq, units):
    offs = inp["offsets"].numpy().astype(np.int64)
    bs = sorted({b for b, _ in units})
    rows, new_offs, remap = [], [0], {}
    for i, b in enumerate(bs):
        remap[b] = i
        rows.append(deq[offs[b]:offs[b + 1]])
        new_offs.append(new_offs[-1] + offs[b + 1] - offs[b])
    o, _ = oracle.decode(np64(inp["q_nope"][bs]), np64(inp["q_rope"][bs]), np.concatenate(rows), new_offs,
                         inp["W_UK"], inp["W_UV"], w.scale, units=[(remap[b], h) for b, h in units], absorbed=True)
    return o


@pytest.mark.parametrize("lengths", [[300, 1, 77, 513, 64], [0, 1000, 2], [4096, 129]])
def test_fp8_decode_matches_the_oracle(lengths):
    """Every (sequence, head) of a few ragged sequences: the FP8 decode against the float64
    decode on the oracle's dequantised rows (the GPU quantises the same bf16 rows; the first
    test holds its bytes to the oracle's)."""
    w, inp = fp8_inputs(lengths, seed=81)
    dims = dims_v3()
    nb = mla.mla_fp8_row_bytes(dims)
    cache = torch.zeros((inp["rows"].shape[0], nb), dtype=torch.uint8, device=DEV)
    mla.mla_quantize_cache_fp8(dims, inp["rows"].to(DEV), cache)
    out = run_fp8_decode(w, inp, cache)
    _, deq = oracle.fp8_rows_f32(inp["rows"], 512, nb)
    units = [(b, h) for b, L in enumerate(lengths) if L > 0 for h in range(w.H)]
    want = oracle_fp8_units(w, inp, deq, units)
    assert_close(torch.stack([out[b, h] for b, h in units]), want, "bf16", f"fp8 decode {lengths}")
    for b, L in enumerate(lengths):
        if L == 0:
            assert torch.all(out[b] == 0)


def test_fp8_decode_full_size_sampled():
    """The V3 decode workload's shape (32 sequences of 4096 tokens) with FP8 rows, sampled
    (sequence, head) units against the oracle."""
    w = V3
    inp = workloads.make_inputs(w)
    dims = dims_v3()
    nb = mla.mla_fp8_row_bytes(dims)
    cache = torch.zeros((inp["cache"].shape[0], nb), dtype=torch.uint8, device=DEV)
    mla.mla_quantize_cache_fp8(dims, inp["cache"].to(DEV), cache)
    inp["rows"] = inp["cache"]
    out = run_fp8_decode(w, inp, cache)
    r = np.random.default_rng(83)
    units = sorted({(int(r.integers(w.B)), int(r.integers(w.H))) for _ in range(40)} | {(0, 0), (w.B - 1, w.H - 1)})
    bs = sorted({b for b, _ in units})
    offs = inp["offsets"].numpy().astype(np.int64)
    deq = np.zeros((int(offs[-1]), w.row))
    for b in bs:
        _, deq[offs[b]:offs[b + 1]] = oracle.fp8_rows_f32(inp["cache"][offs[b]:offs[b + 1]], 512, nb)
    want = oracle_fp8_units(w, inp, deq, units)
    assert_close(torch.stack([out[b, h] for b, h in units]), want, "bf16", "fp8 decode V3 sampled")
