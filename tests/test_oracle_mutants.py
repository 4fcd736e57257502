"""The pins must reject plausible mistakes: each case below plants one mistake
in a copy of oracle.c (on the CPU), builds it, and requires at least one pin of
pins.py to fail on that build."""
import os

import numpy as np
import pytest

import oracle
import pins

MUTANTS = [
    ("nibble_order_swapped",
     "int code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);",
     "int code = (k % 2 == 0) ? (byte >> 4) : (byte & 0x0F);"),
    ("tie_rule_quarter", "if (a <= 0.25f) m = 0;", "if (a < 0.25f) m = 0;"),
    ("tie_rule_five", "else if (a <= 5.0f) m = 6;", "else if (a < 5.0f) m = 6;"),
    ("scale_divisor", "orc_f32_to_bf16_rne(mx / 6.0f)", "orc_f32_to_bf16_rne(mx / 4.0f)"),
    ("encode_drops_sign", "return (r < 0.0f) ? (m | 8) : m;", "return m;"),
    ("decode_table_entry", "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f}",
     "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 5.0f}"),
    ("gate_up_swapped", "double g = gu[i], u = gu[I + i];", "double g = gu[I + i], u = gu[i];"),
    ("silu_sign", "act[i] = g / (1.0 + exp(-g)) * u;", "act[i] = g / (1.0 + exp(g)) * u;"),
    ("router_ties_high", "return a < b;", "return a > b;"),
    ("softmax_drops_term", "for (int j = 0; j < k; ++j) den +=", "for (int j = 1; j < k; ++j) den +="),
    ("combine_unweighted", "y[h] += (double)w[j] * o[h];", "y[h] += o[h];"),
    ("input_reversed", "gu[n] += x[kk] *", "gu[n] += x[H - 1 - kk] *"),
    ("group_unstable", "for (int64_t p = 0; p < P; ++p)\n            if (idx[p] == e) {",
     "for (int64_t p = P - 1; p >= 0; --p)\n            if (idx[p] == e) {"),
    ("bf16_round_half_up", "u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("router_gemm_transposed",
     "(double)orc_bf16_to_f32(w_bf16[(int64_t)e * H + h]);",
     "(double)orc_bf16_to_f32(w_bf16[(int64_t)h * E + e]);"),
    ("router_gemm_drops_last_column", "for (int h = 0; h < H; ++h)\n                acc +=",
     "for (int h = 0; h < H - 1; ++h)\n                acc +="),
    ("router_gemm_first_token_only", "acc += (double)orc_bf16_to_f32(x_bf16[(int64_t)t * H + h]) *",
     "acc += (double)orc_bf16_to_f32(x_bf16[h]) *"),
    ("int2_level_offset", "double orc_int2_decode(int q) { return (double)(q & 3) - 1.5; }",
     "double orc_int2_decode(int q) { return (double)(q & 3) - 1.0; }"),
    ("int2_tie_rule", "    if (r < 0.0f) return 1;\n    if (r < 1.0f) return 2;",
     "    if (r <= 0.0f) return 1;\n    if (r < 1.0f) return 2;"),
    ("int2_bit_order", "codes[(e * (K / 4) + k / 4) * N + n] |= (uint8_t)(q << (2 * (k % 4)));",
     "codes[(e * (K / 4) + k / 4) * N + n] |= (uint8_t)(q << (6 - 2 * (k % 4)));"),
    ("int2_scale_divisor", "orc_f32_to_bf16_rne(mx / 1.5f)", "orc_f32_to_bf16_rne(mx / 2.0f)"),
    ("mixed_ignores_format", "const int f = fmt ? fmt[e] : 0;", "const int f = 0;"),
    ("down_scale_group", "return (float)orc_e2m1_decode(code) * orc_bf16_to_f32(scales[(k / 32) * N + n]);",
     "return (float)orc_e2m1_decode(code) * orc_bf16_to_f32(scales[((k / 32) / 2) * N + n]);"),
    ("e4m3_tie_odd", "if (d < bd || (d == bd && (c & 1) == 0)) {", "if (d < bd || (d == bd && (c & 1) == 1)) {"),
    ("e4m3_bias", "ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    ("nvfp4_row_scale", "const float g = amax / 2688.0f;", "const float g = amax / 1344.0f;"),
    ("nvfp4_block_max_of_first_block", "if (fabsf(v[b * 16 + kk]) > ab) ab = fabsf(v[b * 16 + kk]);",
     "if (fabsf(v[kk]) > ab) ab = fabsf(v[kk]);"),
    ("nvfp4_divides_by_scale_factor_only", "const float rq = (dq > 0.0f) ? 1.0f / dq : 0.0f;",
     "const float rq = (dq > 0.0f) ? 1.0f / (float)orc_e4m3_decode(sb) : 0.0f;"),
    ("nvfp4_act_not_bf16", "af[i] = orc_bf16_to_f32(orc_f64_to_bf16_rne(gv / (1.0 + exp(-gv)) * uv));",
     "af[i] = (float)(gv / (1.0 + exp(-gv)) * uv);"),
    ("nvfp4_down_reads_unencoded_act", "acc += orc_nvfp4_value(ac, as, ga, kk) *", "acc += (double)af[kk] *"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / "oracle_mut.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / f"liboracle_{name}.so"))
    o = oracle.Oracle(lib)
    failed = []
    for cname, check in pins.ALL_CHECKS:
        try:
            check(o, np.random.default_rng(2024))
        except (AssertionError, ValueError):
            failed.append(cname)
    assert failed, f"no pin rejects the planted mistake '{name}'"
