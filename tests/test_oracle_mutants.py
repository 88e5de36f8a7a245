"""Plant plausible mistakes in a copy of the oracle's C source and check that the pins
catch every one of them (CPU only).  The real oracle is never modified."""
import os

import pytest

import oracle
from oracle import build as obuild
import pins

MUTANTS = {
    "rope_sign": ("out[2 * i] = x0 * c - x1 * s;", "out[2 * i] = x0 * c + x1 * s;"),
    "rope_frequency": ("-2.0 * (double)i / (double)d", "-1.0 * (double)i / (double)d"),
    "rope_pairing": ("double x0 = x[2 * i], x1 = x[2 * i + 1];",
                     "double x0 = x[i], x1 = x[i + d / 2];"),
    "drop_positional_term": ("s[t] = scale * (content + positional);", "s[t] = scale * (content);"),
    "drop_scale": ("s[t] = scale * (content + positional);", "s[t] = (content + positional);"),
    "no_softmax_normalisation": ("for (int t = 0; t < T; ++t) s[t] /= l;", ""),
    "v_from_w_uk": ("acc += W_UV_h[(size_t)j * d_c + i] * c[i];", "acc += W_UK_h[(size_t)j * d_c + i] * c[i];"),
    "absorbed_w_uk_transposed": ("for (int j = 0; j < qk_nope; ++j) acc += W_UK_h[(size_t)j * d_c + i] * q_nope[j];",
                                 "for (int j = 0; j < qk_nope; ++j) acc += W_UK_h[(size_t)(i % qk_nope) * d_c + j] * q_nope[j];"),
    "absorbed_o_lat_unweighted": ("o_lat[i] += s[t] * c[i];", "o_lat[i] += c[i] / T;"),
    "query_layout": ("((size_t)hd * qh + j) * d_model", "((size_t)j * H + hd) * d_model"),
    "query_no_rope": ("oracle_rope(d_hR, q + qk_nope, (double)pos[i], theta,", "oracle_rope(d_hR, q + qk_nope, 0.0, theta,"),
    "latent_rope_position": ("oracle_rope(d_hR, kr, (double)pos[i], theta, row + d_c);",
                             "oracle_rope(d_hR, kr, (double)(pos[i] + 1), theta, row + d_c);"),
    "bf16_truncates": ("double r = rint(ldexp(m, 8));", "double r = floor(ldexp(m, 8));"),
    "causal_excludes_self": ("oracle_attend_naive(t + 1, d_c", "oracle_attend_naive(t, d_c"),
    "multi_window_off_by_one": ("- (q_len - 1 - t);   /* keys up to the token itself */",
                                "- (q_len - t);   /* keys up to the token itself */"),
    "multi_query_index": ("size_t q = ((size_t)b * q_len + t) * H + h;", "size_t q = ((size_t)t * q_len + b) * H + h;"),
    "e4m3_truncates": ("double r = rint(a / q) * q;", "double r = floor(a / q) * q;"),
    "e4m3_two_mantissa_bits": ("double q = ldexp(1.0, ue - 3);", "double q = ldexp(1.0, ue - 2);"),
    "e4m3_subnormal_quantum": ("int ue = e - 1 < -6 ? -6 : e - 1;", "int ue = e - 1 < -7 ? -7 : e - 1;"),
    "fp8_scale_to_240": ("double sc = amax > 0.0 ? amax / 448.0 : 1.0;", "double sc = amax > 0.0 ? amax / 240.0 : 1.0;"),
    "mla_row_without_rope": ("return (d_c + d_hR) * layers;", "return d_c * layers;"),
    "rope_pairs_sign": ("y[2 * i] = (float)(p0 - p1);", "y[2 * i] = (float)(p0 + p1);"),
    "rope_pairs_swapped": ("double x0 = x[2 * i], x1 = x[2 * i + 1], c = cs[2 * i], s = cs[2 * i + 1];",
                           "double x1 = x[2 * i], x0 = x[2 * i + 1], c = cs[2 * i], s = cs[2 * i + 1];"),
    "e4m3_bits_bias": ("return (uint8_t)(sign | ((ex + 7) << 3) | mant);", "return (uint8_t)(sign | ((ex + 8) << 3) | mant);"),
    "e4m3_bits_no_sign": ("uint8_t sign = signbit(v) ? 0x80 : 0x00;", "uint8_t sign = 0x00;"),
    "fp8_row_scale_not_stored": ("memcpy(out + d_c + 2 * d_hR, &s, 4);", ""),
    "fp8_row_rope_low_half": ("uint16_t b = (uint16_t)(bits >> 16);", "uint16_t b = (uint16_t)(bits & 0xFFFF);"),
    "fp8_row_scale_to_240": ("float s = amax > 0.0f ? num / den : 1.0f;", "float s = amax > 0.0f ? num / 240.0f : 1.0f;"),
    "out_proj_transposed": ("acc += W_O[(size_t)j * Hv + k] * o[(size_t)i * Hv + k];",
                            "acc += W_O[(size_t)(k % d_model) * Hv + j % Hv] * o[(size_t)i * Hv + k];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(obuild.SRC).read()
    assert old in src, f"mutation site for {name} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(obuild.build(str(path), str(tmp_path / "libmutant.so")))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin detects the mutant {name}"
