"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case plants one mistake -- a wrong rounding rule, a dropped term, a swapped
index or nibble, a wrong constant -- either in a copy of svdq_oracle.c (compiled
on the CPU into a temporary library that replaces the oracle's for the duration
of the case) or in one Python step of the oracle (replaced with pytest's
monkeypatch), then runs the pins named beside it.  At least one of them must
fail with an assertion; a mistake that every named pin lets through is a pin
gap.  The real oracle is never modified, and nothing here touches the CUDA
library."""
import ctypes
import functools
import math

import numpy as np
import pytest

import oracle
import test_oracle_awq as t_awq
import test_oracle_codecs as t_codecs
import test_oracle_dynamic as t_dyn
import test_oracle_gelu as t_gelu
import test_oracle_method as t_method
import test_oracle_w8a8 as t_w8


def _all_golden_points():
    for row in t_codecs._golden():
        t_codecs.test_golden_points(*row)


CODEC_PINS = [_all_golden_points, t_codecs.test_e2m1_bruteforce_dense, t_codecs.test_e2m1_decode_table,
              t_codecs.test_e4m3_against_torch_all_midpoints, t_codecs.test_e4m3_saturates,
              t_codecs.test_fp16_against_numpy, t_codecs.test_bf16_against_torch,
              t_codecs.test_f64_to_bf16_single_rounding]
FWD = [functools.partial(t_method.test_forward_equals_dequantized_matmul, "int4"),
       functools.partial(t_method.test_forward_equals_dequantized_matmul, "nvfp4")]
FWD_NVFP4 = FWD[1:]

# (name, text of svdq_oracle.c, its mistaken replacement, pins expected to catch it)
C_MUTANTS = [
    ("rounding_ties_away_from_zero", "double n = nearbyint(x / quantum);", "double n = round(x / quantum);",
     CODEC_PINS),
    ("bf16_rounded_twice_through_binary32", "double y = rne_to_grid(x, 8, -126);",
     "double y = rne_to_grid((double)(float)x, 8, -126);", [t_codecs.test_f64_to_bf16_single_rounding]),
    ("fp16_subnormal_quantum", "return sign | (uint16_t)(y / ldexp(1.0, -24));",
     "return sign | (uint16_t)(y / ldexp(1.0, -25));", [t_codecs.test_fp16_against_numpy]),
    ("e4m3_no_saturation", "if (y > 448.0 || isinf(y)) y = 448.0;", "if (isinf(y)) y = 448.0;",
     [t_codecs.test_e4m3_saturates, t_codecs.test_e4m3_against_torch_all_midpoints]),
    ("e4m3_subnormal_decode", "else if (e == 0) v = ldexp((double)m, -9);",
     "else if (e == 0) v = ldexp((double)m, -10);", [t_codecs.test_e4m3_against_torch_all_midpoints]),
    ("e2m1_no_saturation", "if (y > 6.0 || isinf(y)) y = 6.0;", "if (isinf(y)) y = 6.0;",
     [t_codecs.test_e2m1_bruteforce_dense]),
    ("e2m1_drops_negative_zero", "if (y == 0.0) return sign;\n  if (y < 1.0) return sign | 0x1;",
     "if (y == 0.0) return 0;\n  if (y < 1.0) return sign | 0x1;", [t_codecs.test_e2m1_bruteforce_dense]),
    ("e2m1_decode_exponent_bias", "ldexp(1.0 + 0.5 * m, e - 1);", "ldexp(1.0 + 0.5 * m, e);",
     [t_codecs.test_e2m1_decode_table]),
    ("smoothing_exponents_swapped", "pow(ax, alpha) / pow(aw, 1.0 - alpha)", "pow(ax, 1.0 - alpha) / pow(aw, alpha)",
     [t_method.test_smoothing_closed_forms]),
    ("smoothing_divides_by_inverse", "volatile float p = x * inv_lambda[k];", "volatile float p = x / inv_lambda[k];",
     [t_method.test_smoothing_preserves_product]),
    ("int4_scale_amax_over_8", "volatile float q7 = amax / 7.0f;", "volatile float q7 = amax / 8.0f;",
     [t_method.test_int4_roundtrip_exact_codes, t_method.test_int4_error_bound_and_zero_group]),
    ("int4_codes_not_clamped", "if (r < -8.0) r = -8.0;\n            if (r > 7.0) r = 7.0;", "",
     [t_method.test_int4_subnormal_scales_saturate_codes]),
    ("int4_nibbles_swapped_on_pack", "(uint8_t)((q[0] & 0xF) | ((q[1] & 0xF) << 4))",
     "(uint8_t)((q[1] & 0xF) | ((q[0] & 0xF) << 4))", [t_method.test_int4_roundtrip_exact_codes]),
    ("int4_nibbles_swapped_on_unpack", "int v = hi ? (byte >> 4) : (byte & 0xF);",
     "int v = hi ? (byte & 0xF) : (byte >> 4);",
     [t_method.test_int4_group_acc_equals_matmul, t_method.test_int4_roundtrip_exact_codes]),
    ("int4_nibble_read_unsigned", "return v >= 8 ? v - 16 : v;", "return v;",
     [t_method.test_int4_group_acc_equals_matmul, t_method.test_int4_roundtrip_exact_codes]),
    ("int4_group_sum_drops_a_term", "for (int64_t k = g * 64; k < g * 64 + 64; ++k)",
     "for (int64_t k = g * 64; k < g * 64 + 63; ++k)", [t_method.test_int4_group_acc_equals_matmul]),
    ("nvfp4_step_without_tensor_scale", "volatile float d = orc_e4m3_to_f32(sb) * g;",
     "volatile float d = orc_e4m3_to_f32(sb);", [t_method.test_nvfp4_roundtrip_on_grid, t_method.test_nvfp4_error_bound]),
    ("nvfp4_block_scale_without_tensor_scale", "const float den = 6.0f * g;", "const float den = 6.0f;",
     [t_method.test_nvfp4_roundtrip_on_grid]),
    ("nvfp4_nibbles_swapped_on_pack", "(uint8_t)(c[0] | (c[1] << 4))", "(uint8_t)(c[1] | (c[0] << 4))",
     [t_method.test_nvfp4_roundtrip_on_grid]),
    ("lowrank_skips_bf16_of_xhat", "double xb = (double)orc_bf16_to_f32(orc_f32_to_bf16(xhat[m * K + k]));",
     "double xb = (double)xhat[m * K + k];", [t_method.test_lowrank_down_matches_matmul]),
    ("lowrank_L1_transposed", "acc[j] += xb * (double)orc_bf16_to_f32(L1[k * r + j]);",
     "acc[j] += xb * (double)orc_bf16_to_f32(L1[j * K + k]);", [t_method.test_lowrank_down_matches_matmul]),
    ("output_drops_bias", "double y = main_ + lr + (bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0);",
     "double y = main_ + lr;", FWD),
    ("output_drops_lowrank_branch", "double y = main_ + lr + (bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0);",
     "double y = main_ + (bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0);", FWD),
    ("output_L2_transposed", "(double)orc_bf16_to_f32(L2[j * N + n]);", "(double)orc_bf16_to_f32(L2[n * r + j]);", FWD),
    ("output_drops_tensor_scales", "if (fmt != 1) main_ = (double)g_x * (double)g_w * main_;", "", FWD_NVFP4),
    ("output_e2m1_factor", "double blk = (fmt == 1) ? (double)s : (double)s * 0.25;",
     "double blk = (fmt == 1) ? (double)s : (double)s * 0.5;", FWD_NVFP4),
    ("output_weight_scales_of_the_wrong_group", "main_ += sxd[m * G + g] * swd[n * G + g] * blk;",
     "main_ += sxd[m * G + g] * swd[n * G + (G - 1 - g)] * blk;", FWD),
    ("rounding_without_the_subnormal_floor", "if (E < emin) E = emin;", "", CODEC_PINS),
    ("e2m1_drops_the_subnormal_half", "if (y < 1.0) return sign | 0x1;", "if (y < 1.0) return sign;",
     [t_codecs.test_e2m1_bruteforce_dense, _all_golden_points]),
    ("fp16_exponent_bias", "return sign | (uint16_t)((E + 15) << 10) | mant;",
     "return sign | (uint16_t)((E + 14) << 10) | mant;", [t_codecs.test_fp16_against_numpy]),
    ("fp16_max_is_overflow", "if (y > 65504.0 || isinf(y)) return sign | 0x7C00;",
     "if (y >= 65504.0 || isinf(y)) return sign | 0x7C00;", [t_codecs.test_fp16_against_numpy, _all_golden_points]),
    ("inverse_lambda_of_the_rounded_lambda", "inv_lambda_f[j] = (float)(1.0 / lam);",
     "inv_lambda_f[j] = 1.0f / (float)lam;", [t_method.test_smoothing_closed_forms]),
    ("int4_group_max_of_signed_values", "for (int i = 0; i < 64; ++i) { float a = fabsf(x[i]);",
     "for (int i = 0; i < 64; ++i) { float a = x[i];", [t_method.test_int4_error_bound_and_zero_group]),
    ("int4_rounds_toward_zero", "double r = nearbyint((double)p);", "double r = trunc((double)p);",
     [t_method.test_int4_error_bound_and_zero_group]),
    ("int4_scale_not_rounded_to_fp16", "float S = orc_f16_to_f32(s);", "float S = q7;",
     [t_method.test_int4_error_bound_and_zero_group, t_method.test_int4_subnormal_scales_saturate_codes]),
    ("nvfp4_block_max_of_signed_values", "for (int i = 0; i < 16; ++i) { float a = fabsf(x[i]);",
     "for (int i = 0; i < 16; ++i) { float a = x[i];", [t_method.test_nvfp4_error_bound]),
    ("nvfp4_zero_scale_block_quantized", "if (sb != 0) {\n          volatile float inv = 1.0f / d;",
     "{\n          volatile float inv = 1.0f / d;", [t_method.test_nvfp4_zero_scale_blocks_have_zero_codes]),
    ("nvfp4_dequant_without_tensor_scale",
     "double d = (double)orc_e4m3_to_f32(scales[m * B + k / 16]) * (double)g;",
     "double d = (double)orc_e4m3_to_f32(scales[m * B + k / 16]);", [t_method.test_nvfp4_roundtrip_on_grid]),
    ("t_rounded_through_binary32", "t[m * r + j] = orc_f64_to_bf16(acc[j]);",
     "t[m * r + j] = orc_f32_to_bf16((float)acc[j]);", [t_method.test_lowrank_down_rounds_once]),
    ("output_rounded_through_binary32", "y_bf16[m * N + n] = orc_f64_to_bf16(y);",
     "y_bf16[m * N + n] = orc_f32_to_bf16((float)y);", [t_method.test_output_rounds_once_from_binary64]),
    ("int4_divides_instead_of_the_reciprocal", "volatile float p = x[i + h] * inv;\n            double r",
     "volatile float p = x[i + h] / S;\n            double r", [t_method.test_int4_code_uses_the_binary32_reciprocal]),
    ("nvfp4_divides_instead_of_the_reciprocal", "volatile float p = x[i + h] * inv;\n            c[h]",
     "volatile float p = x[i + h] / d;\n            c[h]", [t_method.test_nvfp4_code_uses_the_binary32_reciprocal]),
]


def _caught(pins) -> list[str]:
    failed = []
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed.append(getattr(pin, "__name__", None) or pin.func.__name__)
    return failed


def _load_copy(src_text: str, tmp_path, monkeypatch) -> None:
    """Compile `src_text` like the oracle and make it the oracle's library for this test."""
    c = tmp_path / "svdq_oracle_copy.c"
    c.write_text(src_text, encoding="utf-8")
    so = tmp_path / "liboracle_copy.so"
    oracle.compile_source(str(c), str(so))
    monkeypatch.setattr(oracle, "_lib", oracle.bind(ctypes.CDLL(str(so))))


def test_unmodified_copy_passes_every_pin(monkeypatch, tmp_path):
    """Control: the same compile-and-swap path with no mistake planted fails no pin,
    so a failure in the cases below comes from the planted mistake."""
    _load_copy(open(oracle._SRC, encoding="utf-8").read(), tmp_path, monkeypatch)
    pins = {id(p): p for m in C_MUTANTS for p in m[3]}
    assert _caught(list(pins.values())) == []


@pytest.mark.parametrize("name,old,new,pins", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_mistake_in_oracle_c_is_caught(name, old, new, pins, monkeypatch, tmp_path):
    src = open(oracle._SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"{name}: the planted text must occur exactly once in svdq_oracle.c"
    _load_copy(src.replace(old, new), tmp_path, monkeypatch)
    assert _caught(pins), f"mistake '{name}' passed every named pin"


# --------------------------------------------------------------------------- Python steps
def _pow2_scale_one_binade_high(amax):
    a = float(amax) / (oracle.E2M1_MAX * oracle.E4M3_MAX)
    if a <= 0.0:
        return 1.0
    return math.ldexp(1.0, math.frexp(a)[1])  # loses the exact-power-of-two case


def _svd_unbalanced(What, rank):
    L1, L2, S = _REAL["svd_lowrank_factors"](What, rank)
    sq = np.sqrt(S[:rank])
    return L1 * sq[None, :], L2 / sq[:, None], S  # L1 = V S, L2 = U^T: same product, unbalanced


def _smoothed_weight_divides(W_bf16, amax_x, alpha):
    What, lams = _REAL["smoothed_weight"](W_bf16, amax_x, alpha)
    return What / lams[1].astype(np.float64)[None, :] ** 2, lams  # W / lambda instead of W * lambda


def _prepare_residual_from_unrounded_factors(W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd=None):
    out = _REAL["prepare"](W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd)
    if rank:
        What, _ = oracle.smoothed_weight(W_bf16, amax_x, alpha)
        L1d, L2d, _ = oracle.svd_lowrank_factors(What, rank)
        out["R"] = np.ascontiguousarray((What - (L1d @ L2d).T).astype(np.float32))
    return out


def _gelu_wrong_sign(h):
    h = np.asarray(h, np.float64)
    return 0.5 * h * np.vectorize(math.erfc)(h / math.sqrt(2.0))


def _act_tensor_scale_doubled(xhat):
    return 2.0 * _REAL["act_tensor_scale"](xhat)


def _awq_scales_exponent_swapped(mean_abs, alpha):
    return _REAL["awq_channel_scales"](mean_abs, 1.0 - alpha)


def _awq_statistic_max(X_bf16):
    return np.abs(oracle.bf16_to_f32(X_bf16).astype(np.float64)).max(axis=0)


def _quantize_act_t_from_unsmoothed_x(X_bf16, prep):
    act = _REAL["quantize_act"](X_bf16, prep)
    act["t"] = oracle.lowrank_down(oracle.bf16_to_f32(X_bf16), prep["L1"])
    return act


def _prepare_g_w_from_smoothed_weight(W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd=None):
    out = _REAL["prepare"](W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd)
    if oracle._FMT[fmt] == oracle.NVFP4:
        What, _ = oracle.smoothed_weight(W_bf16, amax_x, alpha)
        out["g_w"] = oracle.pow2_scale(float(np.abs(What).max()))
        out["wcodes"], out["wscales"] = oracle.quant_nvfp4(out["R"], out["g_w"])
    return out


def _prepare_static_g_x_unsmoothed(W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd=None):
    out = _REAL["prepare"](W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd)
    if oracle._FMT[fmt] == oracle.NVFP4:
        out["g_x"] = oracle.pow2_scale(float(np.asarray(amax_x, np.float32).max()))
    return out


def _prepare_drops_bias(W_bf16, bias_bf16, amax_x, alpha, rank, fmt, svd=None):
    return _REAL["prepare"](W_bf16, None, amax_x, alpha, rank, fmt, svd)


def _calibration_mean(X_bf16):
    return np.abs(oracle.bf16_to_f32(X_bf16)).mean(axis=0).astype(np.float32)


def _w8_ties_away(v, s):
    v = np.asarray(v, np.float32)
    if s == 0:
        return np.zeros(v.shape, np.int8)
    p = (v * np.float32(np.float32(1.0) / np.float32(s))).astype(np.float64)
    return np.clip(np.sign(p) * np.floor(np.abs(p) + 0.5), -127, 127).astype(np.int8)


def _w8_divides(v, s):
    v = np.asarray(v, np.float32)
    if s == 0:
        return np.zeros(v.shape, np.int8)
    return np.clip(np.rint((v / np.float32(s)).astype(np.float32)), -127, 127).astype(np.int8)


def _w8a8_output_in_binary32(act, prep, want_f64=False):
    acc = act["codes"].astype(np.int64) @ prep["wcodes"].astype(np.int64).T
    yd = (np.float32(act["s_x"]) * np.float32(prep["s_w"]) * acc.astype(np.float32) +
          oracle.bf16_to_f32(prep["bias"])[None, :]).astype(np.float64)
    y = oracle.f64_to_bf16(np.ascontiguousarray(yd))
    return (y, yd) if want_f64 else y


def _awq_smoothed_input_in_binary64(X_bf16, prep, want_f64=False):
    xhat = oracle.bf16_to_f32(X_bf16).astype(np.float64) * prep["inv_s"].astype(np.float64)
    yd = xhat @ oracle.dequant(prep["wcodes"], prep["wscales"], oracle.INT4).T + \
        oracle.bf16_to_f32(prep["bias"]).astype(np.float64)[None, :]
    y = oracle.f64_to_bf16(np.ascontiguousarray(yd))
    return (y, yd) if want_f64 else y


_REAL = {n: getattr(oracle, n) for n in ("svd_lowrank_factors", "smoothed_weight", "prepare", "act_tensor_scale",
                                         "awq_channel_scales", "quantize_act")}

# (name, oracle attribute, its mistaken value, pins expected to catch it)
PY_MUTANTS = [
    ("pow2_scale_one_binade_high", "pow2_scale", _pow2_scale_one_binade_high,
     [t_method.test_pow2_scale, t_method.test_nvfp4_error_bound]),
    ("svd_split_unbalanced", "svd_lowrank_factors", _svd_unbalanced, [t_method.test_svd_recovers_known_spectrum]),
    ("smoothing_divides_the_weight", "smoothed_weight", _smoothed_weight_divides,
     [t_method.test_prepare_residual_uses_rounded_factors]),
    ("residual_from_unrounded_factors", "prepare", _prepare_residual_from_unrounded_factors,
     [t_method.test_prepare_residual_uses_rounded_factors]),
    ("gelu_erfc_sign", "gelu_f64", _gelu_wrong_sign, [t_gelu.test_normal_cdf_points, t_gelu.test_negative_tail]),
    ("dynamic_scale_doubled", "act_tensor_scale", _act_tensor_scale_doubled,
     [t_dyn.test_dynamic_equals_static_calibrated_on_the_same_input]),
    ("w8_step_max_over_126", "W8_QMAX", 126, [functools.partial(t_w8.test_w8_quantizer_properties, 0)]),
    ("awq_scale_exponent_swapped", "awq_channel_scales", _awq_scales_exponent_swapped,
     [t_awq.test_awq_unit_scale_is_plain_group_int4, t_awq.test_awq_exact_layer_equals_dense_product]),
    ("awq_statistic_max_not_mean", "awq_mean_abs", _awq_statistic_max, [t_awq.test_awq_statistic_is_the_channel_mean]),
    ("t_from_the_unsmoothed_input", "quantize_act", _quantize_act_t_from_unsmoothed_x,
     [functools.partial(t_method.test_error_decreases_with_rank_and_full_rank_is_near_exact, "int4")]),
    ("g_w_from_the_smoothed_weight_not_the_residual", "prepare", _prepare_g_w_from_smoothed_weight,
     [t_method.test_tensor_scales_are_tight]),
    ("static_g_x_without_the_smoothing", "prepare", _prepare_static_g_x_unsmoothed,
     [t_method.test_tensor_scales_are_tight, t_dyn.test_dynamic_equals_static_calibrated_on_the_same_input]),
    ("prepare_drops_the_bias", "prepare", _prepare_drops_bias, [t_method.test_prepare_residual_uses_rounded_factors]),
    ("calibration_mean_not_max", "calib_absmax", _calibration_mean,
     [t_dyn.test_dynamic_equals_static_calibrated_on_the_same_input]),
    ("w8_ties_away_from_zero", "quant_w8", _w8_ties_away, [t_w8.test_w8_ties_round_to_even]),
    ("w8_divides_instead_of_the_reciprocal", "quant_w8", _w8_divides,
     [t_w8.test_w8_code_uses_the_binary32_reciprocal]),
    ("w8a8_output_in_binary32", "w8a8_forward_from_act", _w8a8_output_in_binary32,
     [t_w8.test_w8a8_output_rounds_once]),
    ("awq_smoothed_input_in_binary64", "awq_forward", _awq_smoothed_input_in_binary64,
     [t_awq.test_awq_smoothed_input_is_binary32]),
]


def test_python_pins_pass_unmodified():
    """Control for the Python-step cases: their pins pass on the real oracle."""
    pins = {id(p): p for m in PY_MUTANTS for p in m[3]}
    assert _caught(list(pins.values())) == []


@pytest.mark.parametrize("name,attr,value,pins", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_mistake_in_oracle_python_step_is_caught(name, attr, value, pins, monkeypatch):
    assert hasattr(oracle, attr)
    monkeypatch.setattr(oracle, attr, value)
    assert _caught(pins), f"mistake '{name}' passed every named pin"
