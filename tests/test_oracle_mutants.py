"""The pins have teeth: plant one plausible mistake at a time in a copy of the oracle's C
source (on the CPU), rebuild it, and check that at least one pin fails against it."""
import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    "butterfly sign swapped": (
        "v[j + h] = a - b;", "v[j + h] = b - a;",
        [lambda: pins.test_butterfly_matrix_is_sylvester_and_orthogonal(8)]),
    "butterfly partner index off": (
        "float b = v[j + h];", "float b = v[j ^ (h >> 1)];",
        [lambda: pins.test_butterfly_equals_dense_product_on_integers(16)]),
    "normaliser not folded into the scale": (
        "qr[k] = (int8_t)code;\n        }\n        s[r] = s_z * c_g;",
        "qr[k] = (int8_t)code;\n        }\n        s[r] = s_z;",
        [lambda: pins.test_codes_brute_force_g8(16)]),
    "round half away from zero": (
        "float n = nearbyintf(t);", "float n = roundf(t);",
        [lambda: pins.test_codes_brute_force_g8(32),
         lambda: pins.test_g1_is_textbook_per_row_absmax_int8()]),
    "absmax per group instead of per row": (
        "z[k] = bf16_bits_to_f32(xr[k]);\n        for (int64_t k0 = 0; k0 < K; k0 += g)\n            fwht_group_f32(z + k0, g);\n        float amax = 0.0f;\n        for (int64_t k = 0; k < K; k++) {",
        "z[k] = bf16_bits_to_f32(xr[k]);\n        for (int64_t k0 = 0; k0 < K; k0 += g)\n            fwht_group_f32(z + k0, g);\n        float amax = 0.0f;\n        for (int64_t k = 0; k < g; k++) {",
        [lambda: pins.test_golden_worked_rotquant()]),
    "grid 255 levels (range -128..127)": (
        "const float s_z = amax / 127.0f;\n        int8_t *qr = q + r * K;",
        "const float s_z = amax / 127.5f;\n        int8_t *qr = q + r * K;",
        [lambda: pins.test_codes_brute_force_g8(8)]),
    "gemm operand transposed": (
        "const int8_t *bn = b + n * K;", "const int8_t *bn = b + n;",
        [lambda: pins.test_gemm_matches_numpy_int64((17, 33, 48))]),
    "epilogue scale order changed": (
        "float t = sx[m] * sw[n];\n            float v = (float)acc[m * N + n] * t;",
        "float v = ((float)acc[m * N + n] * sx[m]) * sw[n];",
        [lambda: pins.test_epilogue_within_one_ulp_of_fp64_and_op_order()]),
    "epilogue bias add fused into a multiply-add": (
        "(float)acc[m * N + n] * t;\n            if (bias)\n                v = v + bf16_bits_to_f32(bias[n]);",
        "(float)acc[m * N + n] * t;\n            if (bias)\n                v = fmaf((float)acc[m * N + n], t, bf16_bits_to_f32(bias[n]));",
        [lambda: pins.test_epilogue_rounds_twice_not_fused()]),
    "bias dropped": (
        "(float)acc[m * N + n] * t;\n            if (bias)\n                v = v + bf16_bits_to_f32(bias[n]);",
        "(float)acc[m * N + n] * t;\n            if (bias)\n                v = v;",
        [lambda: pins.test_golden_worked_epilogue()]),
    "bf16 rounding truncates": (
        "u += 0x7fffu + lsb;", "u += 0u * lsb;",
        [lambda: pins.test_f32_to_bf16_matches_torch_cast()]),
    "double rounding through fp32": (
        "out[i] = f64_to_bf16_rne(in[i]);", "out[i] = f32_to_bf16_rne((float)in[i]);",
        [lambda: pins.test_f64_to_bf16_is_single_correct_rounding()]),
    "gelu tanh approximation": (
        "double y = 0.5 * x * erfc(-x / sqrt(2.0));",
        "double y = 0.5 * x * (1.0 + tanh(0.7978845608 * (x + 0.044715 * x * x * x)));",
        [lambda: pins.test_gelu_against_scipy_normal_cdf_and_special_values()]),
    "lora B transposed": (
        "(double)bf16_bits_to_f32(B[j * N + n]);", "(double)bf16_bits_to_f32(B[n * rank + j]);",
        [lambda: pins.test_lora_down_and_up_against_fp64_products()]),
    "backward: column scale not folded into dy": (
        "c[n] = bf16_bits_to_f32(dy[r * ld + n]) * sw[n];", "c[n] = bf16_bits_to_f32(dy[r * ld + n]);",
        [lambda: pins.test_grad_input_exact_case_against_explicit_hadamard(64)]),
    "backward: weight codes read transposed": (
        "sum += (int32_t)a[m * N + n] * (int32_t)b[n * K + k];",
        "sum += (int32_t)a[m * N + n] * (int32_t)b[k * N + n];",
        [lambda: pins.test_gemm_nn_matches_numpy_int64()]),
    "backward: rotation not undone": (
        "            fwht_group_f32(z + k0, g);\n        for (int64_t k = 0; k < K; k++)\n            dx[",
        "            (void)k0;\n        for (int64_t k = 0; k < K; k++)\n            dx[",
        [lambda: pins.test_grad_input_exact_case_against_explicit_hadamard(256)]),
    "backward: 1/sqrt(g) dropped": (
        "dx[m * K + k] = f32_to_bf16_rne(z[k] * c_g);", "dx[m * K + k] = f32_to_bf16_rne(z[k]);",
        [lambda: pins.test_grad_input_exact_case_against_explicit_hadamard(256)]),
    "fp8: e4m3 ties away from zero": (
        "double q = nearbyint(a / quantum) * quantum;", "double q = round(a / quantum) * quantum;",
        [lambda: pins.test_e4m3_encode_matches_torch_cast_in_range()]),
    "fp8: int8 grid used for the e4m3 scale": (
        "const float s_z = amax / 448.0f;", "const float s_z = amax / 127.0f;",
        [lambda: pins.test_rotate_quantize_fp8_brute_force(64)]),
    "fp8: subnormal spacing wrong": (
        "if (E < -6)\n        E = -6;", "if (E < -7)\n        E = -7;",
        [lambda: pins.test_e4m3_encode_matches_torch_cast_in_range()]),
    "fp8: products summed in fp32": (
        "            double sum = 0.0;\n            for (int64_t k = 0; k < K; k++)\n                sum += lut[a[m * K + k]] * lut[b[n * K + k]];",
        "            float sum = 0.0f;\n            for (int64_t k = 0; k < K; k++)\n                sum += (float)(lut[a[m * K + k]] * lut[b[n * K + k]]);",
        [lambda: pins.test_fp8_gemm_matches_numpy_fp64()]),
    "attention: channel mean not subtracted from K": (
        "z[d] = bf16_bits_to_f32(k[r * D + d]) - mu[(b * H + h) * D + d];",
        "z[d] = bf16_bits_to_f32(k[r * D + d]);",
        [lambda: pins.test_attn_smooth_k_subtracts_the_exact_channel_mean()]),
    "attention: softmax scale dropped": (
        "logits[bhi * Lk + j] = v * scale;", "logits[bhi * Lk + j] = v;",
        [lambda: pins.test_attn_logits_are_dequantized_products()]),
    "attention: V rows of the wrong head": (
        "const uint16_t *vr = v + ((b * Lk + j) * H + h) * D;",
        "const uint16_t *vr = v + ((b * Lk + j) * H) * D;",
        [lambda: pins.test_attn_softmax_pv_matches_torch_fp64()]),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new, checks = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation site not unique for {name!r}"
    with oracle.built_from(src.replace(old, new), str(tmp_path)):
        caught = 0
        for check in checks:
            try:
                check()
            except (AssertionError, ValueError):
                caught += 1
        assert caught > 0, f"no pin caught the planted mistake: {name}"
