"""Checks that pin the float64 oracle to facts other than itself.

Each pin_* function takes a loaded oracle library (so the mutation test can run the same
checks against deliberately broken copies) and raises AssertionError on failure.  The
facts come from the pages' printed figures (tests/golden/page_figures.json), closed forms,
library routines for special cases (torch's scaled-dot-product attention, numpy matmul and
complex exponentials) and invariants.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_figures.json")


def _rs(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what=""):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.sqrt(np.mean(b * b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} * {scale:.3e}"


def _sdpa(q, k, v, scale, causal=False):
    """torch's attention on float64 CPU tensors: q [Lq, d], k [Lk, d], v [Lk, dv]."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))[None, None]
    out = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale, is_causal=causal)
    return out[0, 0].numpy()


# ------------------------------------------------------------------ page figures

def pin_page_figures(lib):
    g = json.load(open(GOLDEN))
    m = g["mha_kv_bytes_per_token"]
    b = oracle.mha_elems_per_token(m["heads"], m["d_head"], lib) * m["layers"] * m["bytes_per_elem"]
    assert b == m["value_bytes"] == 512 * 1024, b
    c = g["mha_100k_context"]
    gb = b * c["tokens"] / 1e9
    assert abs(gb - c["printed_gb"]) / c["printed_gb"] <= c["rel_tol"], gb
    t = g["memory_table"]
    mha = oracle.mha_elems_per_token(1, t["d_model"], lib)      # H * d_head = d_model
    mla = oracle.mla_elems_per_token(t["d_c"], t["d_hR"], 1, lib)
    assert mha == t["mha_values"] and mla == t["mla_values"], (mha, mla)
    assert math.floor(mha / mla * 10) / 10 == t["printed_ratio"]   # the page truncates 17.78
    mha_gb = mha * t["tokens"] * t["layers"] * t["bytes_per_elem"] / 1e9
    mla_gb = mla * t["tokens"] * t["layers"] * t["bytes_per_elem"] / 1e9
    assert abs(mha_gb - t["printed_mha_gb"]) / t["printed_mha_gb"] <= t["gb_rel_tol"], mha_gb
    assert math.floor(mla_gb * 10) / 10 == t["printed_mla_gb"], mla_gb
    q = g["gqa_equivalence"]
    assert 2 * q["groups"] * q["d_head"] == oracle.mla_elems_per_token(q["d_c"], q["d_hR"], 1, lib)
    v = g["v3_cache_example"]
    e = oracle.mla_elems_per_token(v["kv_lora_rank"], v["qk_rope_head_dim"], v["num_hidden_layers"], lib)
    assert e == v["elements_per_token"], e
    assert e * v["bytes_per_elem"] * v["context"] / 2 ** 30 == v["gib"]


# ------------------------------------------------------------------- rounding

def pin_round_bf16(lib):
    cases = {
        1.0: 0x3F80, -2.5: 0xC020, 0.0: 0x0000,
        1.0 + 2 ** -8: 0x3F80,               # exact tie -> even mantissa (0)
        1.0 + 3 * 2 ** -8: 0x3F82,           # exact tie -> even mantissa (2)
        1.0 + 2 ** -8 + 2 ** -30: 0x3F81,    # just above the tie: one rounding, not two
        2.0 ** -130: 0x0008,                 # subnormal
    }
    for x, want in cases.items():
        got = int(lib.oracle_round_bf16(x))
        assert got == want, f"round_bf16({x!r}) = {got:#06x}, want {want:#06x}"
    # values already in float32: torch's float32 -> bfloat16 cast (nearest-even) agrees
    x = _rs(1).standard_normal(4096).astype(np.float32) * np.float32(7.0)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64), lib), ref)


# ------------------------------------------------------------------------ RoPE

def pin_rope(lib):
    r = _rs(2)
    d = 16
    x = r.standard_normal(d)
    assert np.array_equal(oracle.rope(x, 0.0, 10000.0, lib), x)                 # position 0
    # closed form per pair as a complex rotation z * e^{i pos theta^(-2i/d)}
    for pos in (1.0, 7.0, 4096.0, 8192.0):
        y = oracle.rope(x, pos, 10000.0, lib)
        z = x[0::2] + 1j * x[1::2]
        w = z * np.exp(1j * pos * 10000.0 ** (-2.0 * np.arange(d // 2) / d))
        _close(y[0::2], w.real, 1e-12, "rope real")
        _close(y[1::2], w.imag, 1e-12, "rope imag")
        _close(np.hypot(y[0::2], y[1::2]), np.abs(z), 1e-12, "rope norm")
    # sign convention on one pair: [1, 0] at angle pi/2 -> [0, 1]
    _close(oracle.rope(np.array([1.0, 0.0]), math.pi / 2, 10000.0, lib), [0.0, 1.0], 1e-15, "rope sign")
    # the score of two rotated vectors depends only on the position difference
    q, k = r.standard_normal(d), r.standard_normal(d)
    a = oracle.rope(q, 100.0, 10000.0, lib) @ oracle.rope(k, 37.0, 10000.0, lib)
    b = oracle.rope(q, 163.0, 10000.0, lib) @ oracle.rope(k, 100.0, 10000.0, lib)
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a)), (a, b)


# ---------------------------------------------------------- cache rows / query

def pin_latent_rows(lib):
    r = _rs(3)
    n, d_model, d_c, d_hR = 5, 24, 12, 8
    h = r.standard_normal((n, d_model))
    W_DKV = r.standard_normal((d_c, d_model))
    W_KR = r.standard_normal((d_hR, d_model))
    pos = np.array([0, 1, 5, 100, 4097])
    rows = oracle.latent_rows(h, W_DKV, W_KR, pos, 10000.0, lib)
    assert rows.shape == (n, d_c + d_hR)
    _close(rows[:, :d_c], h @ W_DKV.T, 1e-12, "latent c vs matmul")
    # the rotary part, against the complex-exponential closed form of the rotation
    kr = h @ W_KR.T
    for i, p in enumerate(pos):
        z = kr[i, 0::2] + 1j * kr[i, 1::2]
        w = z * np.exp(1j * p * 10000.0 ** (-2.0 * np.arange(d_hR // 2) / d_hR))
        _close(rows[i, d_c::2], w.real, 1e-12, "k_rope real")
        _close(rows[i, d_c + 1::2], w.imag, 1e-12, "k_rope imag")
    # a unit hidden state picks one column of each weight; at position 0 nothing rotates
    e = np.zeros((1, d_model)); e[0, 3] = 1.0
    row = oracle.latent_rows(e, W_DKV, W_KR, [0], 10000.0, lib)[0]
    assert np.array_equal(row, np.concatenate([W_DKV[:, 3], W_KR[:, 3]]))


def pin_query(lib):
    r = _rs(4)
    H, qk_nope, d_hR, d_model = 3, 4, 6, 10
    W_Q = r.standard_normal((H * (qk_nope + d_hR), d_model))
    e = np.zeros((1, d_model)); e[0, 7] = 1.0
    qn, qr = oracle.query(e, W_Q, [0], H, qk_nope, d_hR, 10000.0, lib)
    col = W_Q[:, 7].reshape(H, qk_nope + d_hR)        # head-major, content rows first
    assert np.array_equal(qn[0], col[:, :qk_nope]) and np.array_equal(qr[0], col[:, qk_nope:])
    h = r.standard_normal((2, d_model))
    qn, qr = oracle.query(h, W_Q, [3, 11], H, qk_nope, d_hR, 10000.0, lib)
    q = (h @ W_Q.T).reshape(2, H, qk_nope + d_hR)
    _close(qn, q[:, :, :qk_nope], 1e-12, "q_nope vs matmul")
    for i, p in enumerate((3, 11)):
        z = q[i, :, qk_nope::2] + 1j * q[i, :, qk_nope + 1::2]
        w = z * np.exp(1j * p * 10000.0 ** (-2.0 * np.arange(d_hR // 2) / d_hR))
        _close(qr[i, :, 0::2], w.real, 1e-12, "q_rope real")
        _close(qr[i, :, 1::2], w.imag, 1e-12, "q_rope imag")


# ------------------------------------------------------------------- decode

def _tiny(seed, T=23, d_c=16, d_hR=8, qk_nope=8, v_head=8):
    r = _rs(seed)
    return dict(q_nope=r.standard_normal(qk_nope), q_rope=r.standard_normal(d_hR),
                rows=r.standard_normal((T, d_c + d_hR)), W_UK_h=r.standard_normal((qk_nope, d_c)) / 4,
                W_UV_h=r.standard_normal((v_head, d_c)) / 4)


def pin_decode_vs_library_attention(lib):
    for seed, T in ((5, 1), (6, 23), (7, 64)):
        a = _tiny(seed, T)
        d_c = a["W_UK_h"].shape[1]
        scale = 1 / math.sqrt(8 + 8)
        o, p, lse = oracle.attend(**a, scale=scale, lib=lib)
        c, kr = a["rows"][:, :d_c], a["rows"][:, d_c:]
        K = np.concatenate([c @ a["W_UK_h"].T, kr], axis=1)
        V = c @ a["W_UV_h"].T
        q = np.concatenate([a["q_nope"], a["q_rope"]])[None]
        _close(o, _sdpa(q, K, V, scale)[0], 1e-12, "decode vs torch sdpa")
        s = scale * (K @ q[0])
        assert abs(lse - float(torch.logsumexp(torch.from_numpy(s), 0))) <= 1e-12 * max(1, abs(lse))
        assert abs(p.sum() - 1.0) <= 1e-12 and np.all(p > 0)


def pin_decode_textbook_reduction(lib):
    """qk_nope = v_head = d_c, W_UK = W_UV = I, q_rope = 0: single-KV-head attention on c."""
    r = _rs(8)
    T, d_c, d_hR = 31, 12, 4
    rows = r.standard_normal((T, d_c + d_hR))
    I = np.eye(d_c)
    qn = r.standard_normal(d_c)
    for absorbed in (False, True):
        o, _, _ = oracle.attend(qn, np.zeros(d_hR), rows, I, I, 0.3, absorbed, lib)
        _close(o, _sdpa(qn[None], rows[:, :d_c], rows[:, :d_c], 0.3)[0], 1e-12, "textbook mqa")


def pin_decode_score_split(lib):
    """score = content + positional: with q_nope = 0 only the rotary keys decide p."""
    a = _tiny(9, 17)
    d_c = a["W_UK_h"].shape[1]
    a["q_nope"] = np.zeros_like(a["q_nope"])
    o, _, _ = oracle.attend(**a, scale=0.25, lib=lib)
    c, kr = a["rows"][:, :d_c], a["rows"][:, d_c:]
    _close(o, _sdpa(a["q_rope"][None], kr, c @ a["W_UV_h"].T, 0.25)[0], 1e-12, "positional only")


def pin_decode_special_cases(lib):
    a = _tiny(10, 1)
    d_c = a["W_UK_h"].shape[1]
    o, p, _ = oracle.attend(**a, scale=0.5, lib=lib)                # one row: p = 1
    _close(o, a["W_UV_h"] @ a["rows"][0, :d_c], 1e-13, "T=1")
    a = _tiny(11, 9)
    a["q_nope"][:] = 0; a["q_rope"][:] = 0                          # zero query: uniform p
    o, p, _ = oracle.attend(**a, scale=0.5, lib=lib)
    _close(p, np.full(9, 1 / 9), 1e-15, "uniform p")
    _close(o, (a["rows"][:, :d_c] @ a["W_UV_h"].T).mean(0), 1e-13, "mean of v")
    a = _tiny(12, 29)                                                # keys are a set
    o1, _, _ = oracle.attend(**a, scale=0.5, lib=lib)
    a["rows"] = a["rows"][_rs(13).permutation(29)]
    o2, _, _ = oracle.attend(**a, scale=0.5, lib=lib)
    _close(o1, o2, 1e-13, "permutation")


def pin_naive_equals_absorbed(lib):
    """Absorption is an exact re-association: naive and absorbed agree in float64."""
    for seed, T, d_c, qk, v in ((14, 40, 16, 8, 8), (15, 3, 32, 12, 20), (16, 129, 64, 32, 32)):
        a = _tiny(seed, T, d_c=d_c, d_hR=16 if d_c == 64 else 8, qk_nope=qk, v_head=v)
        on, pn, ln = oracle.attend(**a, scale=0.2, absorbed=False, lib=lib)
        oa, pa, la = oracle.attend(**a, scale=0.2, absorbed=True, lib=lib)
        _close(on, oa, 1e-10, "naive vs absorbed o")
        _close(pn, pa, 1e-10, "naive vs absorbed p")
        assert abs(ln - la) <= 1e-10 * max(1, abs(ln))


def pin_decode_batch_driver(lib):
    r = _rs(17)
    B, H, d_c, d_hR, qk, v = 3, 2, 16, 8, 8, 8
    lens = [5, 0, 11]
    offs = np.concatenate([[0], np.cumsum(lens)])
    rows = r.standard_normal((offs[-1], d_c + d_hR))
    qn, qr = r.standard_normal((B, H, qk)), r.standard_normal((B, H, d_hR))
    WUK, WUV = r.standard_normal((H, qk, d_c)), r.standard_normal((H, v, d_c))
    o, lse = oracle.decode(qn, qr, rows, offs, WUK, WUV, 0.3, lib=lib)
    for b in range(B):
        for h in range(H):
            rr = rows[offs[b]:offs[b + 1]]
            if len(rr) == 0:
                assert np.all(o[b, h] == 0) and lse[b, h] == -np.inf     # empty sequence
                continue
            d = rr[:, :d_c]
            K = np.concatenate([d @ WUK[h].T, rr[:, d_c:]], 1)
            ref = _sdpa(np.concatenate([qn[b, h], qr[b, h]])[None], K, d @ WUV[h].T, 0.3)[0]
            _close(o[b, h], ref, 1e-12, f"batch b={b} h={h}")


def pin_out_proj(lib):
    r = _rs(18)
    o = r.standard_normal((3, 4, 5))
    W_O = r.standard_normal((7, 20))
    _close(oracle.out_proj(o, W_O, lib), o.reshape(3, 20) @ W_O.T, 1e-12, "out proj")


def pin_prefill(lib):
    r = _rs(19)
    S, d_c, d_hR, qk, v = 13, 16, 8, 8, 12
    rows = r.standard_normal((S, d_c + d_hR))
    qn, qr = r.standard_normal((S, qk)), r.standard_normal((S, d_hR))
    WUK, WUV = r.standard_normal((qk, d_c)) / 4, r.standard_normal((v, d_c)) / 4
    t = np.arange(S)
    c = rows[:, :d_c]
    K = np.concatenate([c @ WUK.T, rows[:, d_c:]], 1)
    ref = _sdpa(np.concatenate([qn, qr], 1), K, c @ WUV.T, 0.3, causal=True)
    for absorbed in (False, True):
        o = oracle.prefill_head(qn, qr, rows, WUK, WUV, 0.3, t, absorbed, lib)
        _close(o, ref, 1e-12, "prefill vs causal sdpa")


def pin_e4m3(lib):
    """FP8 E4M3 rounding against the format's definition and torch's float8_e4m3fn cast."""
    table = [(1.0625, 1.0), (1.1875, 1.25), (2.0 ** -10, 0.0), (3 * 2.0 ** -10, 2.0 ** -8),
             (5 * 2.0 ** -11, 2.0 ** -9), (448.0, 448.0), (464.0, 448.0), (1e6, 448.0), (-0.1, -0.1015625),
             (0.0, 0.0), (240.0, 240.0), (17.0, 16.0), (19.0, 20.0), (2.0 ** -6 * 1.0625, 2.0 ** -6)]
    for x, want in table:
        assert oracle.round_e4m3(np.array([x]), lib)[0] == want, (x, want)
    r = _rs(21)
    # float32-representable inputs (torch's cast may pass through float32) over the whole range
    x = (r.standard_normal(20000) * np.exp2(r.uniform(-12, 8.7, 20000))).astype(np.float32)
    x = np.clip(x, -448, 448).astype(np.float64)
    got = oracle.round_e4m3(x, lib)
    ref = torch.from_numpy(x).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, ref), f"{int((got != ref).sum())} values differ from torch's e4m3 cast"
    big = np.abs(x) >= 2.0 ** -6
    assert np.all(np.abs(got - x)[big] <= 2.0 ** -4 * np.abs(x[big]))       # half an ulp, 3-bit mantissa
    assert np.all(np.abs(got - x)[~big] <= 2.0 ** -10)                        # half the subnormal quantum
    assert np.array_equal(oracle.round_e4m3(got, lib), got)                    # representable values stay


def pin_fp8_latent(lib):
    """Per-token FP8 latent: the largest |c| of a token is code 448 and comes back exactly;
    every value within the format's error; the rotary key untouched; a zero token stays zero."""
    r = _rs(22)
    d_c, d_hR = 64, 8
    rows = r.standard_normal((9, d_c + d_hR)) * np.exp2(r.uniform(-8, 8, (9, 1)))
    rows[4, :d_c] = 0.0
    deq, sc = oracle.quantize_latent_fp8(rows, d_c, lib)
    for t in range(9):
        c, q = rows[t, :d_c], deq[t, :d_c]
        assert np.array_equal(deq[t, d_c:], rows[t, d_c:]), "k_r is not quantised"
        if t == 4:
            assert sc[t] == 1.0 and np.all(q == 0)
            continue
        amax = np.max(np.abs(c))
        assert abs(sc[t] - amax / 448) <= 1e-15 * sc[t]
        codes = q / sc[t]
        assert abs(np.max(np.abs(codes)) - 448.0) <= 1e-12, "the largest element is code 448"
        _close(oracle.round_e4m3(codes, lib), codes, 1e-12, "codes are e4m3 values")
        assert np.all(np.abs(q - c) <= 2.0 ** -4 * np.abs(c) + 2.0 ** -10 * sc[t] * (1 + 1e-12))
    # scaling a token by a power of two scales its codes' scale and nothing else
    deq2, sc2 = oracle.quantize_latent_fp8(rows * 8.0, d_c, lib)
    assert np.array_equal(deq2[:, :d_c], deq[:, :d_c] * 8.0) and np.array_equal(sc2[[0, 1, 2, 3, 5]], sc[[0, 1, 2, 3, 5]] * 8)


def pin_rope_pairs_f32(lib):
    """The float-output rotation: with (cos, sin) of the oracle's own angle it is the oracle's
    float64 RoPE rounded once to float, bit for bit (pairing, signs and order included)."""
    r = _rs(24)
    d, theta = 64, 10000.0
    for pos in (0, 1, 17, 4095, 40000):
        x = r.standard_normal(d).astype(np.float32)
        ang = pos * theta ** (-2.0 * np.arange(d // 2) / d)
        cs = np.stack([np.cos(ang), np.sin(ang)], 1)
        y = oracle.rope_pairs_f32(x, cs, lib)
        ref = oracle.rope(x.astype(np.float64), pos, theta, lib).astype(np.float32)
        assert np.array_equal(y.view(np.uint32), ref.view(np.uint32)), f"pos {pos}"


def pin_e4m3_bits(lib):
    """The E4M3 byte encoding: every finite E4M3 value (all 254 non-NaN patterns) encodes to
    the byte torch's float8_e4m3fn gives it, and a few patterns worked out by hand."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    finite = ~np.isnan(vals)
    got = oracle.e4m3_bits(vals[finite], lib)
    assert np.array_equal(got, codes.numpy()[finite]), "E4M3 bytes differ from torch's encoding"
    for v, byte in [(448.0, 0x7E), (-448.0, 0xFE), (1.0, 0x38), (-0.0, 0x80), (2.0 ** -9, 0x01), (2.0 ** -6, 0x08),
                    (1.125, 0x39), (-0.1015625, 0x9D)]:
        assert int(oracle.e4m3_bits(np.array([v]), lib)[0]) == byte, (v, byte)


def pin_fp8_row_f32(lib):
    """The FP8 cache row with its decisions in float: codes equal torch's float8_e4m3fn cast
    of the float quotients c / s (s = float(amax) / 448 in float), the rotary key is the
    row's bf16 bytes, the scale field holds s, the rest is zero; it differs from the
    float64-decision quantiser only where a quotient's float rounding crosses an E4M3
    rounding boundary."""
    r = _rs(23)
    d_c, d_hR, nb = 64, 8, 96
    rows = r.standard_normal((40, d_c + d_hR)) * np.exp2(r.uniform(-10, 10, (40, 1)))
    rows[3, :d_c] = 0.0
    rows[5, 7] = -0.0
    rows = torch.from_numpy(rows).to(torch.bfloat16).to(torch.float64).numpy()   # bf16-valued rows
    out, deq = oracle.fp8_rows_f32(rows, d_c, nb, lib)
    t = torch.from_numpy(rows).to(torch.float32)
    amax = t[:, :d_c].abs().amax(1)
    s = torch.where(amax > 0, amax / torch.tensor(448.0, dtype=torch.float32), torch.ones_like(amax))
    codes = (t[:, :d_c] / s[:, None]).to(torch.float8_e4m3fn)
    assert np.array_equal(out[:, :d_c], codes.view(torch.uint8).numpy()), "codes differ from torch's float cast"
    kr = t[:, d_c:].to(torch.bfloat16).contiguous().view(torch.uint8).numpy()
    assert np.array_equal(out[:, d_c:d_c + 2 * d_hR], kr), "the rotary key is the row's bf16 bytes"
    assert np.array_equal(out[:, d_c + 2 * d_hR:d_c + 2 * d_hR + 4].copy().view(np.float32)[:, 0], s.numpy())
    assert not out[:, d_c + 2 * d_hR + 4:].any(), "padding is zero"
    assert np.all(out[3, :d_c] == 0) and s[3] == 1.0, "a zero latent: codes 0, scale 1"
    _close(deq[:, :d_c], codes.to(torch.float64).numpy() * s.double().numpy()[:, None], 0.0, "dequantised = code x s")
    assert np.array_equal(deq[:, d_c:], rows[:, d_c:])
    ref, sc64 = oracle.quantize_latent_fp8(rows, d_c, lib)
    assert np.allclose(s.double().numpy(), sc64, rtol=2.0 ** -23, atol=0), "scales agree to float rounding"
    code32 = codes.to(torch.float64).numpy()
    code64 = oracle.round_e4m3(ref[:, :d_c] / sc64[:, None], lib)   # snaps the division's last-bit noise
    same = code32 == code64
    assert same.mean() > 0.99, "codes agree with the float64 decisions except near rounding boundaries"


def pin_decode_multi(lib):
    """Multi-token decode: token t of the q_len new ones attends to the keys up to itself.
    Checked against torch attention with an explicit boolean mask, against the causal
    prefill of the same sequence, and q_len = 1 against the one-token decode."""
    r = _rs(20)
    B, q_len, H, d_c, d_hR, qk, v = 3, 3, 2, 16, 8, 8, 12
    lens = [7, 3, 2]                     # 3 = q_len: the first new token sees one key; 2 < q_len
    offs = np.concatenate([[0], np.cumsum(lens)])
    rows = r.standard_normal((offs[-1], d_c + d_hR))
    qn, qr = r.standard_normal((B, q_len, H, qk)), r.standard_normal((B, q_len, H, d_hR))
    WUK, WUV = r.standard_normal((H, qk, d_c)) / 4, r.standard_normal((H, v, d_c)) / 4
    for absorbed in (False, True):
        o = oracle.decode_multi(qn, qr, rows, offs, WUK, WUV, 0.3, absorbed=absorbed, lib=lib)
        for b in range(B):
            L = lens[b]
            rr = rows[offs[b]:offs[b + 1]]
            c = rr[:, :d_c]
            for h in range(H):
                K = np.concatenate([c @ WUK[h].T, rr[:, d_c:]], 1)
                V = c @ WUV[h].T
                for t in range(q_len):
                    n_keys = L - q_len + t + 1
                    if n_keys <= 0:
                        assert np.all(o[b, t, h] == 0), "a token with no keys gives 0"
                        continue
                    mask = torch.from_numpy(np.arange(L) < n_keys)[None, None, None]
                    q = torch.from_numpy(np.concatenate([qn[b, t, h], qr[b, t, h]]))[None, None, None]
                    ref = torch.nn.functional.scaled_dot_product_attention(
                        q, torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None], attn_mask=mask,
                        scale=0.3)[0, 0, 0].numpy()
                    _close(o[b, t, h], ref, 1e-12, f"multi b={b} t={t} h={h}")
    # the new tokens' outputs are the causal prefill's outputs at their positions
    b, h, L = 0, 1, lens[0]
    QN, QR = r.standard_normal((L, qk)), r.standard_normal((L, d_hR))
    QN[L - q_len:], QR[L - q_len:] = qn[b, :, h], qr[b, :, h]
    pre = oracle.prefill_head(QN, QR, rows[:L], WUK[h], WUV[h], 0.3, list(range(L - q_len, L)), False, lib)
    o = oracle.decode_multi(qn, qr, rows, offs, WUK, WUV, 0.3, absorbed=True, lib=lib)
    _close(o[b, :, h], pre, 1e-12, "multi vs causal prefill")
    # one new token: the one-token decode
    o1 = oracle.decode_multi(qn[:, :1], qr[:, :1], rows, offs, WUK, WUV, 0.3, lib=lib)
    d1, _ = oracle.decode(qn[:, 0], qr[:, 0], rows, offs, WUK, WUV, 0.3, lib=lib)
    _close(o1[:, 0], d1, 1e-13, "q_len = 1")


ALL_PINS = [pin_page_figures, pin_round_bf16, pin_rope, pin_latent_rows, pin_query,
            pin_decode_vs_library_attention, pin_decode_textbook_reduction, pin_decode_score_split,
            pin_decode_special_cases, pin_naive_equals_absorbed, pin_decode_batch_driver,
            pin_out_proj, pin_prefill, pin_decode_multi, pin_e4m3, pin_fp8_latent, pin_e4m3_bits,
            pin_fp8_row_f32, pin_rope_pairs_f32]
