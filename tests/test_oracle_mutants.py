"""The oracle's pins have teeth: plausible mistakes planted in a copy of the
oracle (a dropped term, a wrong sign, index, bias, rounding rule or order of
operations) each make the pin that covers that function fail.

Each mutant of ptpc_oracle.c is compiled by gcc into a temporary library that
the oracle module is pointed at for the duration of one pin; the functions
written in numpy (the attention oracle, the fp64 dot products, the row
selection of the references) are mutated by re-executing their source with
one line changed.
Nothing here touches the CUDA path.  CPU only.
"""
import inspect
import os
import subprocess

import pytest

import oracle
import test_oracle_codec as codec
import test_oracle_gemm as gemm
import test_oracle_quant as quant
import test_oracle_subbyte as subbyte
import synthetic

_C_SRC = os.path.join(os.path.dirname(oracle.__file__), "ptpc_oracle.c")

# (name, original text, planted text, the pin that must fail)
C_MUTANTS = [
    ("decode subnormal exponent", "mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);",
     lambda: codec.test_decode_matches_library_for_all_256_codes()),
    ("decode exponent bias", "mag = ldexp((double)(8 + m), e - 10);", "mag = ldexp((double)(8 + m), e - 11);",
     lambda: codec.test_decode_matches_library_for_all_256_codes()),
    ("encode ties away from zero",
     "if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0))\n        f += 1.0;\n    q = f * step;                          /* rounded",
     "if (rem >= 0.5)\n        f += 1.0;\n    q = f * step;                          /* rounded",
     lambda: codec.test_every_midpoint_rounds_to_even_code()),
    ("encode subnormal threshold", "if (a < ldexp(1.0, -6)) {\n        step = ldexp(1.0, -9);",
     "if (a < ldexp(1.0, -7)) {\n        step = ldexp(1.0, -9);",
     lambda: codec.test_every_midpoint_rounds_to_even_code()),
    ("encode mantissa width", "step = ldexp(1.0, (E - 1) - 3);", "step = ldexp(1.0, (E - 1) - 2);",
     lambda: codec.test_roundtrip_all_finite_codes()),
    ("encode loses the sign of -0", "uint8_t sign = signbit(v) ? 0x80 : 0x00;", "uint8_t sign = (v < 0) ? 0x80 : 0x00;",
     lambda: codec.test_roundtrip_all_finite_codes()),
    ("encode saturates to NaN", "if (q >= E4M3_MAX)\n        return (uint8_t)(sign | 0x7E);",
     "if (q >= E4M3_MAX)\n        return (uint8_t)(sign | 0x7F);",
     lambda: codec.test_every_midpoint_rounds_to_even_code()),
    ("bf16 ties away from zero",
     "if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) == 1.0))\n        f += 1.0;\n    q = f * step;\n    if (q >= ldexp(1.0, 128))",
     "if (rem >= 0.5)\n        f += 1.0;\n    q = f * step;\n    if (q >= ldexp(1.0, 128))",
     lambda: codec.test_bf16_rounding_matches_library_on_fp32_values()),
    ("bf16 subnormal spacing", "step = ldexp(1.0, -133);", "step = ldexp(1.0, -134);",
     lambda: codec.test_bf16_rounding_matches_library_on_fp32_values()),
    ("bf16 infinity pattern", "if (isinf(a))\n        return (uint16_t)(sign | 0x7F80);",
     "if (isinf(a))\n        return (uint16_t)(sign | 0x7F7F);",
     lambda: codec.test_bf16_rounding_fp64_cases()),
    ("scale of a zero group", "if (amax == 0.0f)\n        return 1.0f;", "if (amax == 0.0f)\n        return 0.5f;",
     lambda: quant.test_zero_row_rule()),
    ("scale divisor", "return amax / 448.0f;", "return amax / 447.0f;",
     lambda: quant.test_hand_example_codes_and_scales()),
    ("scale by a reciprocal", "return amax / 448.0f;", "return amax * (1.0f / 448.0f);",
     lambda: quant.test_quant_act_matches_restatement(_x_mix())),
    ("quotient by a reciprocal", "q = x / s;", "q = x * (1.0f / s);",
     lambda: quant.test_quant_act_matches_restatement(_x_mix())),
    ("row maximum without abs", "float a = fabsf(oracle_bf16_to_float(row[k]));", "float a = oracle_bf16_to_float(row[k]);",
     lambda: quant.test_quant_act_matches_restatement(_x_mix())),
    ("weight column read as a row",
     "float a = fabsf(oracle_bf16_to_float(W[k * Co + o]));\n            if (a > amax)\n                amax = a;\n        }\n        s = oracle_scale_from_amax(amax);\n        w_scale[o] = s;",
     "float a = fabsf(oracle_bf16_to_float(W[o * Ci + k]));\n            if (a > amax)\n                amax = a;\n        }\n        s = oracle_scale_from_amax(amax);\n        w_scale[o] = s;",
     lambda: quant.test_weight_quant_is_activation_quant_of_transpose()),
    ("per-tensor maximum over half the tensor", "for (i = 0; i < n; ++i) {\n        float a = fabsf(",
     "for (i = 0; i < n / 2; ++i) {\n        float a = fabsf(",
     lambda: quant.test_per_tensor_is_the_one_token_case()),
    ("naive epilogue scales multiplied first",
     "float v = y[t * Co + o] * x_scale[t];\n            v = v * w_scale[o];",
     "float v = x_scale[t] * w_scale[o];\n            v = v * y[t * Co + o];",
     lambda: gemm.test_fp32_epilogue_rounds_each_product_left_to_right()),
    ("naive epilogue wrong channel", "v = v * w_scale[o];", "v = v * w_scale[t % Co];",
     lambda: gemm.test_naive_two_step_equals_fused()),
    ("fused epilogue scales multiplied first", "float v = (acc * x_scale[t]) * w_scale[o];",
     "float v = acc * (x_scale[t] * w_scale[o]);",
     lambda: gemm.test_fp32_epilogue_overflows_only_in_the_page_order()),
    ("fused epilogue in fp64",
     "float acc = (float)acc64[t * Co + o];\n            float v = (acc * x_scale[t]) * w_scale[o];",
     "double acc = acc64[t * Co + o];\n            float v = (float)((acc * x_scale[t]) * w_scale[o]);",
     lambda: gemm.test_fp32_epilogue_rounds_each_product_left_to_right()),
    ("reference drops the channel scale",
     "double v = (double)x_scale_rows[t] * (double)w_scale[o] * acc64[t * Co + o];",
     "double v = (double)x_scale_rows[t] * acc64[t * Co + o];",
     lambda: gemm.test_reference_epilogue_matches_exact_rational()),
    ("reference rounds through fp32",
     "double v = (double)x_scale_rows[t] * (double)w_scale[o] * acc64[t * Co + o];",
     "double v = (float)((double)x_scale_rows[t] * (double)w_scale[o] * acc64[t * Co + o]);",
     lambda: gemm.test_reference_epilogue_rounds_once()),
    ("E2M1 bias", "case 1: r.ebits = 2; r.mbits = 1; r.bias = 1;", "case 1: r.ebits = 2; r.mbits = 1; r.bias = 2;",
     lambda: subbyte.test_e2m1_values_match_the_ocp_table()),
    ("E3M2 bias", "case 3: r.ebits = 3; r.mbits = 2; r.bias = 3;", "case 3: r.ebits = 3; r.mbits = 2; r.bias = 2;",
     lambda: [subbyte.test_extremes_match_the_ocp_definitions(*c) for c in _extreme_cases()]),
    ("sub-byte sign bit position", "int sign = (code >> nb) & 1;", "int sign = (code >> 7) & 1;",
     lambda: subbyte.test_e2m1_values_match_the_ocp_table()),
    ("sub-byte encoder ties away", "if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) == 1.0))\n            fl += 1.0;",
     "if (rem >= 0.5)\n            fl += 1.0;",
     lambda: subbyte.test_generic_encoder_with_e4m3_parameters_equals_the_pinned_e4m3_encoder()),
    ("sub-byte smallest normal", "min_normal = ldexp(1.0, 1 - t.bias);", "min_normal = ldexp(1.0, - t.bias);",
     lambda: [subbyte.test_encode_roundtrip(f) for f in ("e2m1", "e2m3", "e3m2")]),
    ("FP4 nibble order", "int64_t pos = k * b + bit;", "int64_t pos = (b == 4 ? (k ^ 1) : k) * b + bit;",
     lambda: subbyte.test_packing_against_python_bit_strings("e2m1")),
    ("FP6 bit order", "int64_t pos = k * b + bit;", "int64_t pos = k * b + (b == 6 ? 5 - bit : bit);",
     lambda: subbyte.test_packing_against_python_bit_strings("e2m3")),
    ("split-row maximum without abs",
     "float a = fabsf(oracle_bf16_to_float(X[t * Ci + k]));\n            if (a > m)",
     "float a = oracle_bf16_to_float(X[t * Ci + k]);\n            if (a > m)",
     lambda: quant.test_row_split_quantisation_equals_whole_rows()),
]


def _x_mix():
    return synthetic.with_edge_rows(synthetic.make_x(synthetic.LLAMA8B_PREFILL, 0, 64, 4096))


def _extreme_cases():
    marks = [m for m in subbyte.test_extremes_match_the_ocp_definitions.pytestmark if m.name == "parametrize"]
    return [tuple(c) for c in marks[0].args[1]]


@pytest.fixture(scope="module")
def c_source():
    return open(_C_SRC).read()


@pytest.mark.parametrize("name,orig,planted,pin", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_planted_c_mistake_fails_its_pin(name, orig, planted, pin, c_source, tmp_path, monkeypatch):
    assert c_source.count(orig) == 1, name
    src = tmp_path / "mutant.c"
    lib = tmp_path / "mutant.so"
    src.write_text(c_source.replace(orig, planted))
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
                           "-shared", "-std=c11", str(src), "-o", str(lib), "-lm"])
    pin()                                       # the pin holds on the oracle itself
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "_LIB_PATH", str(lib))
    monkeypatch.setattr(oracle, "_SRC", str(src))
    try:
        with pytest.raises(AssertionError):
            pin()
    finally:
        monkeypatch.setattr(oracle, "_lib", None)


PY_MUTANTS = [
    ("decode_attention_reference", "query head mapped modulo", "g = h // group", "g = h % Hkv"),
    ("decode_attention_reference", "softmax scale dropped",
     "s = softmax_scale * (K[:, g, :] @ q[b, h])", "s = (K[:, g, :] @ q[b, h])"),
    ("decode_attention_reference", "block offset shifted", "offs = pos % block_size", "offs = (pos + 1) % block_size"),
    ("decode_attention_reference", "last context position dropped",
     "pos = np.arange(L)", "pos = np.arange(max(L - 1, 1))"),
    ("decode_attention_reference", "values scaled by the key scales",
     "V = dec[v_codes[blocks, offs]] * v_scales", "V = dec[v_codes[blocks, offs]] * k_scales"),
    ("decode_attention_reference", "negative block entries read (from the end of the cache)",
     "keep = (blocks >= 0) & (blocks < num_blocks)", "keep = blocks < num_blocks"),
    ("decode_attention_reference", "positions past the table read from its last entry",
     "blocks = np.where(bi < len(table), table[np.minimum(bi, len(table) - 1)], -1)",
     "blocks = np.where(True, table[np.minimum(bi, len(table) - 1)], -1)"),
    ("kv_quantize", "heads and tokens swapped",
     "q, s = quant_act(np.ascontiguousarray(KV_bits).reshape(T * H, D))",
     "q, s = quant_act(np.ascontiguousarray(KV_bits.transpose(1, 0, 2)).reshape(T * H, D))"),
    ("gemm_acc64", "weight codes reversed along K",
     "acc[:, o0:o0 + col_chunk] = A @ B.T", "acc[:, o0:o0 + col_chunk] = A @ B[:, ::-1].T"),
    ("gemm_acc64_fmt", "sub-byte codes decoded as E4M3",
     "acc[:, o0:o0 + col_chunk] = A @ dec[codes_t[o0:o0 + col_chunk]].T",
     "acc[:, o0:o0 + col_chunk] = A @ e4m3_decode_table()[codes_t[o0:o0 + col_chunk]].T"),
    ("scaled_mm_reference_fmt", "token scales not following the chosen rows",
     "slice(None) if rows is None else np.asarray(rows)])", "slice(None) if rows is None else np.asarray(rows)[::-1]])"),
    ("fused_f32", "token scales not following the chosen rows",
     "slice(None) if rows is None else np.asarray(rows)])", "slice(None) if rows is None else np.asarray(rows)[::-1]])"),
    ("linear_reference_fmt", "one token scale for all tokens",
     "return scaled_mm_reference_fmt(Xq, xs, codes_t, w_scale, fmt, rows), Xq, xs",
     "return scaled_mm_reference_fmt(Xq, np.full_like(xs, xs.max()), codes_t, w_scale, fmt, rows), Xq, xs"),
]

PY_PINS = {
    "decode_attention_reference": lambda: (gemm.test_decode_attention_oracle_matches_library_attention(),
                                           gemm.test_decode_attention_oracle_edge_cases()),
    "kv_quantize": lambda: gemm.test_kv_cache_oracle(),
    "gemm_acc64": lambda: gemm.test_hand_example_gemm(),
    "gemm_acc64_fmt": lambda: subbyte.test_gemm_exact_against_integer_dot_products("e2m1"),
    "scaled_mm_reference_fmt": lambda: subbyte.test_reference_row_subset_equals_full_rows("e3m2"),
    "fused_f32": lambda: gemm.test_row_subset_equals_full_rows(),
    "linear_reference_fmt": lambda: subbyte.test_generic_reference_with_e4m3_equals_the_ptpc_reference(),
}


@pytest.mark.parametrize("fn,name,orig,planted", PY_MUTANTS, ids=[f"{m[0]}: {m[1]}" for m in PY_MUTANTS])
def test_planted_python_mistake_fails_its_pin(fn, name, orig, planted, monkeypatch):
    pin = PY_PINS[fn]
    src = inspect.getsource(getattr(oracle, fn))
    assert src.count(orig) == 1, name
    ns = dict(vars(oracle))
    exec(src.replace(orig, planted), ns)
    pin()                                       # the pin holds on the oracle itself
    monkeypatch.setattr(oracle, fn, ns[fn])
    with pytest.raises(AssertionError):
        pin()
