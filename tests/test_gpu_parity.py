"""Parity of the CUDA path (through the C ABI) with the float64 oracle, on the same seeded
inputs: reduced sizes that span several tiles and a ragged tail, the full workload sizes on
sampled outputs, and the edge cases (empty, single-row and ragged sequences, B = 0, n = 0,
slots outside the cache).  Invalid offsets and the timeout path are in test_gpu_errors.py."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import CACHE_ABS_RMS, CACHE_EXACT_FRAC, assert_close, bf16_bits, bf16_ulp_diff, np64, rms, to_dev

pytestmark = pytest.mark.gpu

mla = pytest.importorskip("compressed_kv_cache_absorbed_b200")

DEV = "cuda"


def dims_of(w: workloads.Workload):
    return mla.make_dims(w.H, w.d_model, w.d_c, w.d_hR, w.qk_nope, w.v_head, w.dtype)


def storage_round(rows64: np.ndarray, dtype: str) -> np.ndarray:
    """The oracle's cache rows rounded once to the storage type (nearest-even)."""
    if dtype == "f32":
        return rows64.astype(np.float32).astype(np.float64)
    return oracle.bf16_value(oracle.round_bf16(rows64))


def sample_units(B, H, n, seed, must_b=(), must_h=(0,)):
    r = np.random.default_rng(seed)
    units = {(int(b), int(h)) for b in must_b for h in must_h}
    units |= {(0, 0), (0, H - 1)}
    while len(units) < n:
        units.add((int(r.integers(B)), int(r.integers(H))))
    return sorted(units)


# ----------------------------------------------------------------------- append

def check_rows(gpu_rows: torch.Tensor, want64: np.ndarray, dtype: str, what: str):
    if dtype == "f32":
        assert_close(gpu_rows, want64, "f32", what)
        return 1.0
    got = bf16_bits(gpu_rows)
    ref = oracle.round_bf16(want64)
    ulp = bf16_ulp_diff(got, ref)
    # beyond one ulp only where the value is so small that fp32 accumulation error over the
    # d_model-long dot product (~sqrt(K) * 2^-24 * RMS) exceeds a bf16 ulp of it
    err = np.abs(oracle.bf16_value(got) - want64)
    far = (ulp > 1) & (err > CACHE_ABS_RMS * rms(want64))
    assert not far.any(), f"{what}: {int(far.sum())} elements off by more than 1 ulp and the fp32 bound"
    frac = float((ulp == 0).mean())
    assert frac >= CACHE_EXACT_FRAC, f"{what}: only {frac:.4f} of values bit-exact"
    return frac


@pytest.mark.parametrize("name,n", [("tiny_fp32_layer", 37), ("v3_layer_b128_ctx8192", 128),
                                    ("v2_prefill_b4_s4096", 200), ("v2_prefill_b4_s4096", 1300)])
def test_append_rows_and_layout(name, n):
    """n = 1300 takes the token-major GEMM orientation (a thread per token, 16-byte row
    stores, rotary pairs inside one thread); the others the weights-major one."""
    w = workloads.WORKLOADS[name]
    d = workloads.make_weights(w)
    dims = dims_of(w)
    tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    h = torch.from_numpy(np.random.default_rng(1).standard_normal((n, w.d_model))).to(tdt)
    cap = 3 * n + 5
    rng = np.random.default_rng(2)
    slots = np.sort(rng.choice(cap, n, replace=False))[::-1].copy()   # scattered, descending
    pos = rng.integers(0, 40000, n).astype(np.int32)
    pos[0] = 0
    sentinel = torch.full((cap, w.row), -7.25, dtype=tdt)
    cache = sentinel.clone().to(DEV)
    mla.mla_append_cache(dims, h.to(DEV), d["W_DKV"].to(DEV), d["W_KR"].to(DEV),
                         torch.from_numpy(pos).to(DEV), torch.from_numpy(slots).to(DEV), cache)
    assert mla.mla_get_device_error() == (0, 0)
    cache = cache.cpu()
    want = oracle.latent_rows(h, d["W_DKV"], d["W_KR"], pos, w.rope_theta)
    frac = check_rows(cache[torch.from_numpy(slots)], want, w.dtype, f"{name} rows")
    assert frac >= CACHE_EXACT_FRAC
    untouched = np.setdiff1d(np.arange(cap), slots)
    assert torch.equal(cache[torch.from_numpy(untouched)], sentinel[torch.from_numpy(untouched)])


def test_rope_rotation_is_bit_exact():
    """The rotation every rotating kernel applies (cache append, query projection), alone:
    float pairs and given (cos, sin), against the oracle's restatement in IEEE double with
    each operation rounded, bit for bit (values over 40 binades, angles of any size)."""
    r = np.random.default_rng(91)
    n = 64 * 1000
    x = (r.standard_normal(n) * np.exp2(r.uniform(-20, 20, n))).astype(np.float32)
    ang = r.uniform(-1e4, 1e4, n // 2)
    cs = np.ascontiguousarray(np.stack([np.cos(ang), np.sin(ang)], 1))
    y = torch.empty(n, dtype=torch.float32, device=DEV)
    mla.mla_rope_apply(torch.from_numpy(x).to(DEV), torch.from_numpy(cs).to(DEV), y)
    want = oracle.rope_pairs_f32(x, cs)
    got = y.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), \
        f"{int((got.view(np.uint32) != want.view(np.uint32)).sum())} values differ"


def test_append_slot_out_of_range_latches_and_skips():
    w = workloads.WORKLOADS["tiny_fp32_layer"]
    d = workloads.make_weights(w)
    dims = dims_of(w)
    h = torch.randn(4, w.d_model)
    cache = torch.zeros(4, w.row, device=DEV)
    slot = torch.tensor([0, 9, 2, -1], dtype=torch.int64, device=DEV)
    pos = torch.zeros(4, dtype=torch.int32, device=DEV)
    mla.mla_append_cache(dims, h.to(DEV), d["W_DKV"].to(DEV), d["W_KR"].to(DEV), pos, slot, cache)
    st, _ = mla.mla_get_device_error()
    assert st == mla.MLA_ERR_OUT_OF_RANGE
    c = cache.cpu()
    assert torch.all(c[1] == 0) and torch.all(c[3] == 0) and not torch.all(c[0] == 0)
    assert mla.mla_get_device_error() == (0, 0)      # reading clears the word


def test_append_zero_tokens_is_a_noop():
    w = workloads.WORKLOADS["tiny_fp32_layer"]
    cache = torch.zeros(2, w.row, device=DEV)
    e = torch.empty(0, device=DEV)
    mla.mla_append_cache(dims_of(w), e.view(0, w.d_model), e, e, e.int(), e.long(), cache)
    assert torch.all(cache == 0)


# ----------------------------------------------------------------------- decode

def run_decode_attn(w, inp, B=None):
    dims = dims_of(w)
    g = to_dev({k: inp[k] for k in ("cache", "offsets", "q_nope", "q_rope", "W_UK", "W_UV")})
    B = g["offsets"].numel() - 1
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    out = torch.empty(B, w.H, w.v_head, dtype=g["cache"].dtype, device=DEV)
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, B))
    mla.mla_decode_absorbed(dims, weights, g["cache"], g["offsets"], out, ws, q_nope=g["q_nope"],
                            q_rope=g["q_rope"])
    assert mla.mla_get_device_error() == (0, 0)
    return out.cpu()


def oracle_decode_units(w, inp, units, absorbed=True, seqs=None):
    """Oracle o for (b, h) units, reading only the rows of the sequences involved."""
    offs = inp["offsets"].numpy().astype(np.int64)
    bs = sorted({b for b, _ in units})
    rows, new_offs, remap = [], [0], {}
    for i, b in enumerate(bs):
        remap[b] = i
        rows.append(np64(inp["cache"][offs[b]:offs[b + 1]]))
        new_offs.append(new_offs[-1] + offs[b + 1] - offs[b])
    rows = np.concatenate(rows) if rows else np.zeros((0, w.row))
    qn = np64(inp["q_nope"][bs])
    qr = np64(inp["q_rope"][bs])
    o, _ = oracle.decode(qn, qr, rows, new_offs, inp["W_UK"], inp["W_UV"], w.scale,
                         units=[(remap[b], h) for b, h in units], absorbed=absorbed)
    return o


def reduced_attn_inputs(lengths, seed=11):
    w = workloads.WORKLOADS["v3_decode_b32_ctx4096"]
    w = workloads.shrink(w, B=len(lengths), seed=seed)
    d = workloads.make_weights(w)
    r = np.random.default_rng(seed)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    tot = int(offs[-1])
    d["offsets"] = torch.from_numpy(offs)
    d["cache"] = (torch.from_numpy(r.standard_normal((tot, w.row))) * 0.5).to(torch.bfloat16)
    d["q_nope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.qk_nope))).to(torch.bfloat16)
    d["q_rope"] = torch.from_numpy(r.standard_normal((w.B, w.H, w.d_hR))).to(torch.bfloat16)
    return w, d


@pytest.mark.parametrize("lengths", [[300, 1, 77, 513, 64], [0, 1000, 2], [4096, 129]])
def test_decode_attn_reduced_all_units(lengths):
    w, inp = reduced_attn_inputs(lengths)
    out = run_decode_attn(w, inp)
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    want = oracle_decode_units(w, inp, units).reshape(w.B, w.H, w.v_head)
    for b, L in enumerate(lengths):
        if L == 0:
            assert torch.all(out[b] == 0), "an empty sequence decodes to zeros"
    nz = [b for b, L in enumerate(lengths) if L > 0]
    assert_close(out[nz], want[nz], "bf16", f"decode {lengths}")
    # a few units through the naive (materialised K/V) form as well
    few = [(nz[0], 0), (nz[-1], w.H - 1), (nz[0], 77)]
    naive = oracle_decode_units(w, inp, few, absorbed=False)
    assert_close(torch.stack([out[b, h] for b, h in few]), naive, "bf16", "decode vs naive")


@pytest.mark.parametrize("name", ["v3_decode_b32_ctx4096", "v3_ragged_b64"])
def test_decode_attn_full_size_sampled(name):
    w = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(w)
    out = run_decode_attn(w, inp)
    L = workloads.lengths(w)
    must = (int(np.argmax(L)), int(np.argmin(L)), w.B - 1)
    units = sample_units(w.B, w.H, 64, 5, must_b=must, must_h=(0, w.H - 1))
    want = oracle_decode_units(w, inp, units)
    got = torch.stack([out[b, h] for b, h in units])
    assert_close(got, want, "bf16", name)
    naive = oracle_decode_units(w, inp, units[:2], absorbed=False)
    assert_close(got[:2], naive, "bf16", name + " naive")


# --------------------------------------------------------------- decode layer

def run_decode_layer(w, inp, fold=False):
    dims = dims_of(w)
    g = to_dev(inp)
    B = w.B
    offs = inp["offsets"].numpy().astype(np.int64)
    L = workloads.lengths(w)
    if w.history == "hidden":
        cache = torch.zeros(int(offs[-1]), w.row, dtype=g["h_new"].dtype, device=DEV)
        pos = np.tile(np.arange(w.ctx), B).astype(np.int32)
        slot = (offs[:-1, None] + np.arange(w.ctx)[None]).reshape(-1)
        mla.mla_append_cache(dims, g["h_hist"].reshape(-1, w.d_model), g["W_DKV"], g["W_KR"],
                             torch.from_numpy(pos).to(DEV), torch.from_numpy(slot).to(DEV), cache)
    else:
        cache = g["cache"]
    # the token being decoded: appended at position L, then attends over L + 1 rows
    q_pos = torch.from_numpy(L.astype(np.int32)).to(DEV)
    slot = torch.from_numpy(offs[:-1] + L).to(DEV)
    mla.mla_append_cache(dims, g["h_new"], g["W_DKV"], g["W_KR"], q_pos, slot, cache)
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"], g["W_Q"], g["W_O"], fold=fold)
    out = torch.empty(B, w.d_model, dtype=g["h_new"].dtype, device=DEV)
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, B))
    mla.mla_decode_absorbed(dims, weights, cache, g["offsets"], out, ws, h=g["h_new"], q_pos=q_pos)
    assert mla.mla_get_device_error() == (0, 0)
    return out.cpu(), cache


def oracle_decode_layer(w, inp, bs, absorbed):
    """Oracle out[b] for the sequences bs, computing every row it needs itself."""
    L = workloads.lengths(w)
    offs = inp["offsets"].numpy().astype(np.int64)
    rows_all, o_offs = [], [0]
    for b in bs:
        if w.history == "hidden":
            hist = oracle.latent_rows(inp["h_hist"][b], inp["W_DKV"], inp["W_KR"], np.arange(w.ctx), w.rope_theta)
            hist = storage_round(hist, w.dtype)
        else:
            hist = np64(inp["cache"][offs[b]:offs[b] + L[b]])
        new = oracle.latent_rows(inp["h_new"][b:b + 1], inp["W_DKV"], inp["W_KR"], [L[b]], w.rope_theta)
        rows_all.append(np.concatenate([hist, storage_round(new, w.dtype)]))
        o_offs.append(o_offs[-1] + L[b] + 1)
    qn, qr = oracle.query(inp["h_new"][bs], inp["W_Q"], L[bs], w.H, w.qk_nope, w.d_hR, w.rope_theta)
    o, _ = oracle.decode(qn, qr, np.concatenate(rows_all), o_offs, inp["W_UK"], inp["W_UV"], w.scale,
                         absorbed=absorbed)
    return oracle.out_proj(o, inp["W_O"]), np.concatenate([r[-1:] for r in rows_all])


def test_decode_layer_tiny_fp32_end_to_end():
    w = workloads.WORKLOADS["tiny_fp32_layer"]
    inp = workloads.make_inputs(w)
    out, cache = run_decode_layer(w, inp)
    want, _ = oracle_decode_layer(w, inp, list(range(w.B)), absorbed=False)
    assert_close(out, want, "f32", "tiny fp32 layer (naive oracle)")
    # every cache row the GPU wrote (history and new token) against the oracle's rows
    offs = inp["offsets"].numpy()
    for b in range(w.B):
        rows = oracle.latent_rows(np.concatenate([np64(inp["h_hist"][b]), np64(inp["h_new"][b:b + 1])]),
                                  inp["W_DKV"], inp["W_KR"], np.arange(w.ctx + 1), w.rope_theta)
        assert_close(cache[offs[b]:offs[b + 1]].cpu(), rows, "f32", f"tiny cache b={b}")


def test_decode_layer_v3_full_size_sampled():
    w = workloads.WORKLOADS["v3_layer_b128_ctx8192"]
    inp = workloads.make_inputs(w)
    out, cache = run_decode_layer(w, inp)
    bs = [0, 57, w.B - 1]
    want, new_rows = oracle_decode_layer(w, inp, bs, absorbed=True)
    assert_close(out[bs], want, "bf16", "v3 layer out")
    offs = inp["offsets"].numpy().astype(np.int64)
    L = workloads.lengths(w)
    # the appended rows of all 128 sequences, and the untouched history around them
    allnew = oracle.latent_rows(inp["h_new"], inp["W_DKV"], inp["W_KR"], L, w.rope_theta)
    got = cache[torch.from_numpy(offs[:-1] + L).to(DEV)].cpu()
    frac = check_rows(got, allnew, "bf16", "v3 appended rows")
    assert frac >= CACHE_EXACT_FRAC
    assert torch.equal(cache[:8192].cpu(), inp["cache"][:8192])


def test_decode_layer_folded_weights():
    """fold = 1: W_UK folded into W_Q and W_UV into W_O ("Coste de computo", precomputed
    products).  The layer output is the same attention, so it is held to the oracle's layer
    at the same bound: every sequence of a reduced V3-shaped layer (ragged, several tiles), on
    the folded kernels (no q absorption, no W_UV product), and sampled sequences at full size."""
    w = workloads.shrink(workloads.WORKLOADS["v3_layer_b128_ctx8192"], B=5, ctx=300, seed=95)
    inp = workloads.make_inputs(w)
    mla.mla_profile_report(reset=True)
    mla.mla_profile_enable(True)
    try:
        out, _ = run_decode_layer(w, inp, fold=True)
    finally:
        mla.mla_profile_enable(False)
    names = set(mla.mla_profile_report(reset=True))
    assert {"tc_q_lat_folded", "tc_q_rope_folded", "tc_flash_decode", "tc_merge", "tc_w_o_folded"} <= names, names
    assert not names & {"tc_q_absorb", "tc_merge_w_uv", "tc_q_proj_rope", "tc_w_o"}, names
    want, _ = oracle_decode_layer(w, inp, list(range(w.B)), absorbed=True)
    assert_close(out, want, "bf16", "folded layer (reduced)")

    w = workloads.WORKLOADS["v3_layer_b128_ctx8192"]
    inp = workloads.make_inputs(w)
    out, _ = run_decode_layer(w, inp, fold=True)
    bs = [0, 57, w.B - 1]
    want, _ = oracle_decode_layer(w, inp, bs, absorbed=True)
    assert_close(out[bs], want, "bf16", "folded v3 layer out")


# ---------------------------------------------------------------------- prefill

def run_prefill(w, inp):
    dims = dims_of(w)
    g = to_dev(inp)
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"], g["W_Q"])
    cache = torch.zeros(w.B * w.ctx, w.row, dtype=g["h"].dtype, device=DEV)
    out = torch.empty(w.B, w.ctx, w.H, w.v_head, dtype=g["h"].dtype, device=DEV)
    ws = mla.workspace(mla.mla_prefill_workspace_size(dims, w.B, w.ctx))
    mla.mla_prefill_causal(dims, weights, g["h"], g["W_DKV"], g["W_KR"], cache, out, ws)
    assert mla.mla_get_device_error() == (0, 0)
    return out.cpu(), cache.cpu()


def oracle_prefill(w, inp, b, t_list, heads, absorbed=True):
    S_needed = max(t_list) + 1
    rows = oracle.latent_rows(inp["h"][b, :S_needed], inp["W_DKV"], inp["W_KR"], np.arange(S_needed),
                              w.rope_theta)
    rows_s = storage_round(rows, w.dtype)
    qn, qr = oracle.query(inp["h"][b, t_list], inp["W_Q"], t_list, w.H, w.qk_nope, w.d_hR, w.rope_theta)
    # scatter the sampled queries into position-indexed arrays for the per-head routine
    QN = np.zeros((S_needed, w.qk_nope))
    QR = np.zeros((S_needed, w.d_hR))
    res = {}
    for h in heads:
        QN[t_list] = qn[:, h]
        QR[t_list] = qr[:, h]
        res[h] = oracle.prefill_head(QN, QR, rows_s, inp["W_UK"][h], inp["W_UV"][h], w.scale, t_list,
                                     absorbed)
    return res, rows


@pytest.mark.parametrize("B,S", [(2, 200), (2, 1), (1, 128), (3, 257)])
def test_prefill_reduced(B, S):
    """Several query blocks with a ragged last one; one token (one query, one key); exactly
    one block; one query alone in the last block."""
    w = workloads.shrink(workloads.WORKLOADS["v2_prefill_b4_s4096"], B=B, ctx=S, seed=77)
    inp = workloads.make_inputs(w)
    out, cache = run_prefill(w, inp)
    t_list = sorted({t for t in (0, 1, 63, 64, 65, 127, 128, 150, 191, 192, 199, 255, 256) if t < S} | {S - 1})
    heads = [0, 5, 127]
    for b in range(B):
        res, rows = oracle_prefill(w, inp, b, t_list, heads)
        for h in heads:
            assert_close(out[b, t_list, h], res[h], "bf16", f"prefill b={b} h={h}")
        assert len(rows) == S
        check_rows(cache[b * S:(b + 1) * S], rows, "bf16", "prefill cache")
    tn = sorted({0, min(150, S - 1)})
    res, _ = oracle_prefill(w, inp, B - 1, tn, [3], absorbed=False)
    assert_close(out[B - 1, tn, 3], res[3], "bf16", "prefill naive")


def test_prefill_token_major_projections():
    """1100 tokens: the query, K and V projections run token-major; 9 query blocks with a
    ragged last one."""
    w = workloads.shrink(workloads.WORKLOADS["v2_prefill_b4_s4096"], B=1, ctx=1100, seed=79)
    inp = workloads.make_inputs(w)
    out, cache = run_prefill(w, inp)
    t_list = [0, 1, 127, 128, 500, 1023, 1024, 1098, 1099]
    heads = [0, 33, 127]
    res, rows = oracle_prefill(w, inp, 0, t_list, heads)
    for h in heads:
        assert_close(out[0, t_list, h], res[h], "bf16", f"prefill token-major h={h}")
    check_rows(cache[:1100], rows, "bf16", "prefill cache token-major")


def test_prefill_every_query_of_one_head():
    """Every query position of a 3-block sequence (ragged last block) for one head, so each
    row of the causal mask and each block boundary is checked."""
    w = workloads.shrink(workloads.WORKLOADS["v2_prefill_b4_s4096"], B=1, ctx=300, seed=78)
    inp = workloads.make_inputs(w)
    out, _ = run_prefill(w, inp)
    t_list = list(range(300))
    res, _ = oracle_prefill(w, inp, 0, t_list, [77])
    assert_close(out[0, t_list, 77], res[77], "bf16", "prefill every query")


def test_prefill_full_size_sampled():
    w = workloads.WORKLOADS["v2_prefill_b4_s4096"]
    inp = workloads.make_inputs(w)
    out, cache = run_prefill(w, inp)
    b = 2
    t_list = [0, 1, 2, 127, 128, 2047, 4094, 4095]
    heads = [0, 64, 127]
    res, rows = oracle_prefill(w, inp, b, t_list, heads)
    for h in heads:
        assert_close(out[b, t_list, h], res[h], "bf16", f"prefill full h={h}")
    frac = check_rows(cache[b * w.ctx:(b + 1) * w.ctx], rows, "bf16", "prefill cache rows")
    assert frac >= CACHE_EXACT_FRAC


# ------------------------------------------------ split-KV scheduling edge cases

def test_decode_path_is_tensor_core_for_the_v3_head_shape():
    w = workloads.WORKLOADS["v3_decode_b32_ctx4096"]
    assert mla.mla_decode_path(dims_of(w)) == 1


@pytest.mark.parametrize("lengths", [
    [20000],                                   # one sequence split across every cluster
    [1] * 200 + [20000] + [63, 64, 65],        # B > 256 rows of the planner, many pieces per range
    [129, 191, 192, 193, 4095, 1, 2, 3],       # tile-boundary lengths
])
def test_decode_split_schedules(lengths):
    w, inp = reduced_attn_inputs(lengths, seed=31)
    out = run_decode_attn(w, inp)
    r = np.random.default_rng(4)
    units = sorted({(int(r.integers(w.B)), int(r.integers(w.H))) for _ in range(48)} |
                   {(int(np.argmax(lengths)), 0), (int(np.argmax(lengths)), w.H - 1), (w.B - 1, 5)})
    want = oracle_decode_units(w, inp, units)
    assert_close(torch.stack([out[b, h] for b, h in units]), want, "bf16", f"schedule {len(lengths)} seqs")


def test_decode_invariant_to_cache_row_order():
    """Attention over a sequence is a function of its set of (already rotated) rows: with the
    rows of every sequence permuted, the result still matches the oracle (which is order
    invariant).  The two GPU results are each held to the oracle rather than to each other:
    both are rounded to bf16, so they may differ by a bf16 ulp."""
    lengths = [700, 1300, 65]
    w, inp = reduced_attn_inputs(lengths, seed=41)
    out1 = run_decode_attn(w, inp)
    offs = inp["offsets"].numpy()
    perm = np.concatenate([offs[b] + np.random.default_rng(b).permutation(lengths[b]) for b in range(len(lengths))])
    inp2 = dict(inp)
    inp2["cache"] = inp["cache"][torch.from_numpy(perm)].contiguous()
    out2 = run_decode_attn(w, inp2)
    units = [(b, h) for b in range(w.B) for h in range(w.H)]
    want = oracle_decode_units(w, inp, units).reshape(w.B, w.H, w.v_head)
    assert_close(out1, want, "bf16", "rows in order")
    assert_close(out2, want, "bf16", "rows permuted")


# --------------------------------------------- which kernels run (no silent fallback)

def test_v3_bf16_paths_run_the_tensor_core_kernels():
    """A reduced V3-shaped decode layer and prefill: the library's per-launch profile names
    show the tcgen05 kernels ran for every projection and for the attention chain."""
    w = workloads.shrink(workloads.WORKLOADS["v3_layer_b128_ctx8192"], B=3, ctx=70, seed=91)
    inp = workloads.make_inputs(w)
    mla.mla_profile_report(reset=True)
    mla.mla_profile_enable(True)
    try:
        out, _ = run_decode_layer(w, inp)
    finally:
        mla.mla_profile_enable(False)
    names = set(mla.mla_profile_report(reset=True))
    assert {"tc_append_proj_rope", "tc_q_proj_rope", "tc_q_absorb", "tc_flash_decode", "tc_merge_w_uv",
            "tc_w_o"} <= names, names
    assert not any(n.startswith("simt_") for n in names), names
    want, _ = oracle_decode_layer(w, inp, [0, 2], absorbed=True)
    assert_close(out[[0, 2]], want, "bf16", "reduced v3 layer")

    p = workloads.shrink(workloads.WORKLOADS["v2_prefill_b4_s4096"], B=1, ctx=130, seed=92)
    pin = workloads.make_inputs(p)
    mla.mla_profile_enable(True)
    try:
        run_prefill(p, pin)
    finally:
        mla.mla_profile_enable(False)
    names = set(mla.mla_profile_report(reset=True))
    assert {"tc_append_proj_rope", "tc_q_proj_rope", "tc_k_materialise", "tc_v_materialise",
            "tc_prefill_attn"} <= names, names
    assert not any(n.startswith("simt_") for n in names), names


# ------------------------------------------------------------ host-buffer decode

def test_decode_with_host_buffers_matches_the_oracle_and_the_device_call():
    w, inp = reduced_attn_inputs([300, 1, 77, 513, 64], seed=23)
    dims = dims_of(w)
    g = to_dev({k: inp[k] for k in ("cache", "offsets", "W_UK", "W_UV")})
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, w.B))
    qn_h = inp["q_nope"].contiguous().pin_memory()
    qr_h = inp["q_rope"].contiguous().pin_memory()
    out_h = torch.empty(w.B, w.H, w.v_head, dtype=torch.bfloat16).pin_memory()
    mla.mla_decode_absorbed_host(dims, weights, g["cache"], g["offsets"], qn_h, qr_h, out_h, ws)
    torch.cuda.synchronize()
    assert mla.mla_get_device_error() == (0, 0)
    dev = run_decode_attn(w, inp)
    assert torch.equal(out_h, dev), "the host-buffer call runs the same kernels on the same data"
    units = [(b, h) for b in range(w.B) for h in (0, 31, 127)]
    want = oracle_decode_units(w, inp, units)
    assert_close(torch.stack([out_h[b, h] for b, h in units]), want, "bf16", "host-buffer decode")


# -------------------------------------------------------------------- paged cache

def test_paged_cache_gives_the_contiguous_result():
    """The same rows laid out in 64-token pages (random page order, junk in the unused tail
    of each last page, spare pages): bit-identical to the contiguous decode, which the other
    tests hold to the oracle."""
    lengths = [300, 1, 77, 513, 0, 64, 4096, 129]
    w, inp = reduced_attn_inputs(lengths, seed=31)
    dev = run_decode_attn(w, inp)
    r = np.random.default_rng(31)
    npg = [(L + 63) // 64 for L in lengths]
    total_pages = sum(npg) + 5
    perm = r.permutation(total_pages)
    pages = (torch.from_numpy(r.standard_normal((total_pages, 64, w.row))) * 3.0).to(torch.bfloat16)
    max_blocks = max(npg) + 2
    table = np.zeros((w.B, max_blocks), dtype=np.int32)
    offs = inp["offsets"].numpy()
    k = 0
    for b, L in enumerate(lengths):
        for j in range(npg[b]):
            p = int(perm[k])
            k += 1
            table[b, j] = p
            n = min(64, L - 64 * j)
            pages[p, :n] = inp["cache"][offs[b] + 64 * j: offs[b] + 64 * j + n]
    dims = dims_of(w)
    g = to_dev({k_: inp[k_] for k_ in ("q_nope", "q_rope", "W_UK", "W_UV")})
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, w.B))
    out = torch.empty(w.B, w.H, w.v_head, dtype=torch.bfloat16, device=DEV)
    mla.mla_decode_absorbed_paged(dims, weights, pages.to(DEV), torch.from_numpy(table).to(DEV),
                                  torch.tensor(lengths, dtype=torch.int32, device=DEV), out, ws,
                                  q_nope=g["q_nope"], q_rope=g["q_rope"])
    assert mla.mla_get_device_error() == (0, 0)
    out = out.cpu()
    assert torch.equal(out, dev)
    # and directly against the oracle, on the rows as the pages hold them
    units = [(b, h) for b, L in enumerate(lengths) if L > 0 for h in (0, 64, 127)]
    want = oracle_decode_units(w, inp, units)
    assert_close(torch.stack([out[b, h] for b, h in units]), want, "bf16", "paged decode vs oracle")
    assert torch.all(out[lengths.index(0)] == 0)


# ------------------------------------------------------------ multi-token decode

@pytest.mark.parametrize("q_len", [3, 1, 8, 12])
def test_multi_token_decode_over_pages_matches_the_oracle(q_len):
    """q_len new tokens per sequence over a paged cache (random page order, spare pages):
    token t of sequence b attends to the keys up to its own position.  Sequences of 3 and 2
    tokens give new tokens with no key (zeros).  q_len <= 8 runs the queries of a sequence
    on sibling clusters; 12 expands every token into a sequence of its own."""
    lengths = [300, 3, 2, 513, 64, 130]
    w, inp = reduced_attn_inputs(lengths, seed=53)
    r = np.random.default_rng(53)
    qn = torch.from_numpy(r.standard_normal((w.B, q_len, w.H, w.qk_nope))).to(torch.bfloat16)
    qr = torch.from_numpy(r.standard_normal((w.B, q_len, w.H, w.d_hR))).to(torch.bfloat16)
    npg = [(L + 63) // 64 for L in lengths]
    total_pages = sum(npg) + 3
    perm = r.permutation(total_pages)
    pages = torch.zeros(total_pages, 64, w.row, dtype=torch.bfloat16)
    max_blocks = max(npg) + 1
    table = np.zeros((w.B, max_blocks), dtype=np.int32)
    offs = inp["offsets"].numpy()
    k = 0
    for b, L in enumerate(lengths):
        for j in range(npg[b]):
            p = int(perm[k])
            k += 1
            table[b, j] = p
            n = min(64, L - 64 * j)
            pages[p, :n] = inp["cache"][offs[b] + 64 * j: offs[b] + 64 * j + n]
    dims = dims_of(w)
    g = to_dev({k_: inp[k_] for k_ in ("W_UK", "W_UV")})
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    ws = mla.workspace(mla.mla_decode_multi_workspace_size(dims, w.B, q_len, max_blocks))
    out = torch.empty(w.B, q_len, w.H, w.v_head, dtype=torch.bfloat16, device=DEV)
    mla.mla_decode_absorbed_paged_multi(dims, weights, pages.to(DEV), torch.from_numpy(table).to(DEV),
                                        torch.tensor(lengths, dtype=torch.int32, device=DEV), out, ws,
                                        q_nope=qn.to(DEV), q_rope=qr.to(DEV))
    assert mla.mla_get_device_error() == (0, 0)
    out = out.cpu()
    for b, L in enumerate(lengths):
        for t in range(q_len):
            if L - q_len + t + 1 <= 0:
                assert torch.all(out[b, t] == 0), "a new token with no key decodes to zeros"
    units = [(b, t, h) for b in range(w.B) for t in range(q_len) for h in (0, 45, 127)
             if lengths[b] - q_len + t + 1 > 0]
    want = oracle.decode_multi(qn, qr, inp["cache"], inp["offsets"], inp["W_UK"], inp["W_UV"], w.scale,
                               units=units, absorbed=True)
    assert_close(torch.stack([out[b, t, h] for b, t, h in units]), want, "bf16", "multi-token decode")


@pytest.mark.parametrize("chunk,prefix", [(100, [300, 77]), (1000, [4096])])
def test_chunked_prefill_over_an_existing_cache(chunk, prefix):
    """Absorbed chunked prefill: a chunk of new tokens per sequence attends to a cached
    prefix and causally to itself, K and V never materialised: the multi-token call with
    q_len = the chunk (one query sequence per new token).  100-token chunks over 300- and
    77-token prefixes, and a 1000-token chunk over a 4096-token prefix.  Sampled tokens of
    the chunk against the oracle, whose multi-token decode is pinned to its causal prefill."""
    lengths = [p + chunk for p in prefix]
    w, inp = reduced_attn_inputs(lengths, seed=59)
    r = np.random.default_rng(59)
    qn = torch.from_numpy(r.standard_normal((w.B, chunk, w.H, w.qk_nope))).to(torch.bfloat16)
    qr = torch.from_numpy(r.standard_normal((w.B, chunk, w.H, w.d_hR))).to(torch.bfloat16)
    npg = [(L + 63) // 64 for L in lengths]
    pages = torch.zeros(sum(npg), 64, w.row, dtype=torch.bfloat16)
    table = np.zeros((w.B, max(npg)), dtype=np.int32)
    offs = inp["offsets"].numpy()
    perm = r.permutation(sum(npg))
    k = 0
    for b, L in enumerate(lengths):
        for j in range(npg[b]):
            p = int(perm[k])
            k += 1
            table[b, j] = p
            n = min(64, L - 64 * j)
            pages[p, :n] = inp["cache"][offs[b] + 64 * j: offs[b] + 64 * j + n]
    dims = dims_of(w)
    g = to_dev({k_: inp[k_] for k_ in ("W_UK", "W_UV")})
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    ws = mla.workspace(mla.mla_decode_multi_workspace_size(dims, w.B, chunk, table.shape[1]))
    out = torch.empty(w.B, chunk, w.H, w.v_head, dtype=torch.bfloat16, device=DEV)
    mla.mla_decode_absorbed_paged_multi(dims, weights, pages.to(DEV), torch.from_numpy(table).to(DEV),
                                        torch.tensor(lengths, dtype=torch.int32, device=DEV), out, ws,
                                        q_nope=qn.to(DEV), q_rope=qr.to(DEV))
    assert mla.mla_get_device_error() == (0, 0)
    out = out.cpu()
    ts = sorted({0, 1, 63, 64, chunk // 2, chunk - 2, chunk - 1})
    units = [(b, t, h) for b in range(w.B) for t in ts for h in (0, 64, 127)]
    want = oracle.decode_multi(qn, qr, inp["cache"], inp["offsets"], inp["W_UK"], inp["W_UV"], w.scale,
                               units=units, absorbed=True)
    assert_close(torch.stack([out[b, t, h] for b, t, h in units]), want, "bf16", f"chunked prefill {chunk}")


def test_decode_large_batch_spans_several_sequence_blocks():
    """B = 200 short ragged sequences: the q-absorb kernel runs two blocks of 128 sequences
    and the merge kernel four blocks of 64; sampled units against the oracle."""
    r = np.random.default_rng(47)
    lengths = [int(x) for x in r.integers(0, 300, size=200)]
    lengths[0], lengths[129], lengths[199] = 0, 1, 299
    w, inp = reduced_attn_inputs(lengths, seed=47)
    out = run_decode_attn(w, inp)
    units = [(b, h) for b in (1, 63, 64, 127, 128, 129, 150, 199) for h in (0, 77, 127)]
    want = oracle_decode_units(w, inp, units)
    assert_close(torch.stack([out[b, h] for b, h in units]), want, "bf16", "decode B=200")
    assert torch.all(out[0] == 0)
