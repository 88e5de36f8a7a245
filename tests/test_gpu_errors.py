"""The device-side error paths the C ABI promises, on a B200: sequences whose rows are not
inside the cache, and a bounded wait that runs out.  None of these faults or hangs the GPU:
invalid sequences are skipped by every role of the decode kernels (no CTA aborts), and the
timeout test starves the single-CTA projection GEMM of its loads, so that its MMA and
epilogue waits give up with no copy and no MMA in flight."""
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


def attn_inputs(lengths, seed):
    w = workloads.shrink(workloads.WORKLOADS["v3_decode_b32_ctx4096"], B=len(lengths), seed=seed)
    d = workloads.make_weights(w)
    r = np.random.default_rng(seed)
    tot = int(sum(lengths))
    d["cache"] = (torch.from_numpy(r.standard_normal((tot, w.row))) * 0.5).to(torch.bfloat16)
    d["q_nope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.qk_nope))).to(torch.bfloat16)
    d["q_rope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.d_hR))).to(torch.bfloat16)
    return w, d


def decode(w, inp, offsets, cache_rows=None):
    dims = mla.make_dims(w.H, w.d_model, w.d_c, w.d_hR, w.qk_nope, w.v_head, w.dtype)
    cache = inp["cache"] if cache_rows is None else inp["cache"][:cache_rows]
    weights = mla.mla_absorb_weights(dims, inp["W_UK"].to(DEV), inp["W_UV"].to(DEV))
    B = len(offsets) - 1
    out = torch.full((B, w.H, w.v_head), 3.0, dtype=torch.bfloat16, device=DEV)
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, B))
    mla.mla_decode_absorbed(dims, weights, cache.contiguous().to(DEV),
                            torch.tensor(offsets, dtype=torch.int32, device=DEV), out, ws,
                            q_nope=inp["q_nope"][:B].to(DEV), q_rope=inp["q_rope"][:B].to(DEV))
    st = mla.mla_get_device_error()
    weights.close()
    return out.cpu(), st


def oracle_seq(w, inp, b, r0, r1, heads=(0, 64, 127)):
    rows = np64(inp["cache"][r0:r1])
    o, _ = oracle.decode(np64(inp["q_nope"][b:b + 1]), np64(inp["q_rope"][b:b + 1]), rows, [0, r1 - r0],
                         inp["W_UK"], inp["W_UV"], w.scale, units=[(0, h) for h in heads], absorbed=True)
    return o


@pytest.mark.parametrize("case", ["decreasing", "negative", "past_cache_rows"])
def test_invalid_sequences_latch_and_decode_to_zero(case):
    """A sequence whose rows are not inside the cache latches MLA_ERR_OUT_OF_RANGE and decodes
    to zeros; the valid sequences of the same call still match the oracle, and the next call
    with valid offsets is clean."""
    lengths = [300, 77, 513, 64]
    w, inp = attn_inputs(lengths, seed=61)
    good = [0, 300, 377, 890, 954]
    cache_rows = None
    if case == "decreasing":
        offs = [0, 300, 200, 890, 954]          # sequence 1 ends before it starts
        bad = [1]
    elif case == "negative":
        offs = [-64, 300, 377, 890, 954]        # sequence 0 starts before the cache
        bad = [0]
    else:
        offs = good
        cache_rows = 900                        # sequence 3 (rows 890 .. 953) runs past the cache
        bad = [3]
    out, (st, _) = decode(w, inp, offs, cache_rows)
    assert st == mla.MLA_ERR_OUT_OF_RANGE
    for b in bad:
        assert torch.all(out[b] == 0), f"invalid sequence {b} decodes to zeros"
    heads = (0, 64, 127)
    for b in range(len(lengths)):
        if b in bad:
            continue
        want = oracle_seq(w, inp, b, offs[b], offs[b + 1], heads)
        assert_close(torch.stack([out[b, h] for h in heads]), want, "bf16", f"{case}: valid sequence {b}")
    # the error word was cleared by reading it; a valid call afterwards is clean and correct
    out2, st2 = decode(w, inp, good)
    assert st2 == (0, 0)
    want = oracle_seq(w, inp, 2, 377, 890, heads)
    assert_close(torch.stack([out2[2, h] for h in heads]), want, "bf16", f"{case}: next call")


def test_a_wait_that_runs_out_latches_a_timeout_and_the_next_call_works():
    """The projection GEMM of a bf16 cache append is starved of its loads (test hook) with a
    short wait limit: its waits give up, the call latches MLA_ERR_DEVICE_TIMEOUT and writes
    no row.  With the hook off and the default limit restored, the same append writes the
    oracle's rows."""
    r = np.random.default_rng(67)
    dm, n = 256, 5
    dims = mla.make_dims(128, dm, 512, 64, 128, 128, "bf16")
    h = torch.from_numpy(r.standard_normal((n, dm))).to(torch.bfloat16)
    W_DKV = torch.from_numpy(r.standard_normal((512, dm)) / 16).to(torch.bfloat16)
    W_KR = torch.from_numpy(r.standard_normal((64, dm)) / 16).to(torch.bfloat16)
    pos = torch.tensor([0, 1, 7, 100, 4095], dtype=torch.int32)
    slot = torch.tensor([6, 0, 3, 1, 5], dtype=torch.int64)
    sentinel = torch.full((8, 576), -7.25, dtype=torch.bfloat16)
    g = {k: v.to(DEV) for k, v in dict(h=h, W_DKV=W_DKV, W_KR=W_KR, pos=pos, slot=slot).items()}
    assert mla.mla_get_device_error() == (0, 0)
    cache = sentinel.clone().to(DEV)
    mla.mla_set_wait_limit(256)
    mla.mla_test_starve_projection(True)
    try:
        mla.mla_append_cache(dims, g["h"], g["W_DKV"], g["W_KR"], g["pos"], g["slot"], cache)
        st, detail = mla.mla_get_device_error()
    finally:
        mla.mla_test_starve_projection(False)
        mla.mla_set_wait_limit(0)
    assert st == mla.MLA_ERR_DEVICE_TIMEOUT, (st, detail)
    assert torch.equal(cache.cpu(), sentinel), "a starved projection writes nothing"
    # the context is usable and the kernels are whole again
    cache = sentinel.clone().to(DEV)
    mla.mla_append_cache(dims, g["h"], g["W_DKV"], g["W_KR"], g["pos"], g["slot"], cache)
    assert mla.mla_get_device_error() == (0, 0)
    rows = oracle.latent_rows(h, W_DKV, W_KR, pos.numpy())
    got = cache.cpu().double().numpy()[slot.numpy()]
    assert np.all(np.abs(got - rows) <= 2.0 ** -7 * np.abs(rows) + 1e-3)
    untouched = [2, 4, 7]
    assert torch.equal(cache.cpu()[untouched], sentinel[untouched])
