"""Planted mistakes in the oracle must fail its pins.

Each case edits a copy of oracle/msda_oracle.c (a dropped term, a wrong sign
or index, a transposed operand, a wrong pixel convention), builds it into a
temporary directory, swaps it in for the real oracle and runs the pin checks,
expecting at least one of them to fail.  Every mutant keeps its memory
accesses inside the arrays.  CPU only; nothing runs on a GPU.
"""
import contextlib
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_dcn as dcn_pins
from tests import test_oracle_fp8 as fp8_pins
from tests import test_oracle_linear as linear_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "msda_oracle.c")
_PIX = "return bilinear_at_pixel(lx * (double)W - 0.5, ly * (double)H - 0.5, H, W);"

MUTATIONS = {
    "no_half_pixel_shift": (_PIX, "return bilinear_at_pixel(lx * (double)W, ly * (double)H - 0.5, H, W);"),
    "align_corners_true": (_PIX, "return bilinear_at_pixel(lx * (double)(W - 1), ly * (double)H - 0.5, H, W);"),
    "x_y_swapped_scale": (_PIX, "return bilinear_at_pixel(lx * (double)W - 0.5, ly * (double)W - 0.5, H, W);"),
    "corner_weight_transposed": ("s.w[1] = (1.0 - s.fy) * s.fx;", "s.w[1] = s.fy * (1.0 - s.fx);"),
    "column_mirrored": ("int64_t key = start_l + cy * W + cx;",
                        "int64_t key = start_l + cy * W + (W - 1 - cx);"),
    "level_start_ignored": ("int64_t key = start_l + cy * W + cx;", "int64_t key = cy * W + cx;"),
    # clamping corners to the border (the other option the pages mention)
    # instead of masking them to zero; every access stays inside the map
    "border_clamp_not_zero": ("s.inb[c] = s.cx[c] >= 0 && s.cx[c] < W && s.cy[c] >= 0 && s.cy[c] < H;",
                              "s.cx[c] = s.cx[c] < 0 ? 0 : (s.cx[c] >= W ? W - 1 : s.cx[c]); "
                              "s.cy[c] = s.cy[c] < 0 ? 0 : (s.cy[c] >= H ? H - 1 : s.cy[c]); "
                              "s.inb[c] = 1;"),
    "grad_x_scale_H": ("grad_loc[2 * p] = (double)W * a * gx;", "grad_loc[2 * p] = (double)H * a * gx;"),
    "dsdx_sign": ("  double dx = (1.0 - s.fy) * (v01 - v00) + s.fy * (v11 - v10);",
                  "  double dx = (1.0 - s.fy) * (v00 - v01) + s.fy * (v11 - v10);"),
    "dsdy_dropped_term": ("  double dy = (1.0 - s.fx) * (v10 - v00) + s.fx * (v11 - v01);",
                          "  double dy = (1.0 - s.fx) * (v10 - v00);"),
    "grad_value_no_weight": ("gv[ch] += a * s.w[c] * g[ch];", "gv[ch] += a * g[ch];"),
    "grad_attn_unweighted": ("  double samp = s.w[0] * v00 + s.w[1] * v01 + s.w[2] * v10 + s.w[3] * v11;",
                             "  double samp = v00 + v01 + v10 + v11;"),
    "offset_normalizer_swapped": ("loc[2 * p] = r[0] + off[2 * p] / (double)shapes[2 * l + 1];",
                                  "loc[2 * p] = r[0] + off[2 * p] / (double)shapes[2 * l];"),
    "softmax_no_normalize": ("a[j] /= sum;", "a[j] /= 1.0;"),
    "softmax_jacobian_sign": ("grad_logits[r * n + j] = attn[r * n + j] * (grad_attn[r * n + j] - dot);",
                              "grad_logits[r * n + j] = attn[r * n + j] * (grad_attn[r * n + j] + dot);"),
    "grad_off_not_scaled": ("grad_off[2 * p] = grad_loc[2 * p] / (double)shapes[2 * l + 1];",
                            "grad_off[2 * p] = grad_loc[2 * p];"),
    "grad_ref_y_from_x": ("grad_ref[2 * (b * d->Q + q) + 1] += grad_loc[2 * p + 1];",
                          "grad_ref[2 * (b * d->Q + q) + 1] += grad_loc[2 * p];"),
}

# mistakes in the DCNv3 core, caught by its own pins
DCN_MUTATIONS = {
    "dcn_no_dilation": ("const double px = (double)(j * d->stride_w - d->pad_w + c * d->dil_w) + dp[0];",
                        "const double px = (double)(j * d->stride_w - d->pad_w + c) + dp[0];"),
    "dcn_offset_xy_swapped": ("const double py = (double)(i * d->stride_h - d->pad_h + r * d->dil_h) + dp[1];",
                              "const double py = (double)(i * d->stride_h - d->pad_h + r * d->dil_h) + dp[0];"),
    "dcn_grid_transposed": ("const int64_t r = k / d->kw, c = k % d->kw;",
                            "const int64_t c = k / d->kh, r = k % d->kh;"),
    "dcn_grad_offset_unweighted": ("grad_offset[2 * p] = mask[p] * gx;", "grad_offset[2 * p] = gx;"),
    "dcn_grad_x_no_mask": ("gxr[ch] += mask[p] * s.w[c] * gy[ch];", "gxr[ch] += s.w[c] * gy[ch];"),
    "dcn_stride_ignored": ("const double py = (double)(i * d->stride_h - d->pad_h + r * d->dil_h) + dp[1];",
                           "const double py = (double)(i - d->pad_h + r * d->dil_h) + dp[1];"),
}

# mistakes in the dense layer and the query head, caught by their own pins
LINEAR_MUTATIONS = {
    "linear_weight_transposed": ("s += x[r * K + k] * w[n * K + k];", "s += x[r * K + k] * w[(k * N + n) % (N * K)];"),
    "linear_bias_dropped": ("double s = b ? b[n] : 0.0;", "double s = 0.0;"),
    "linear_grad_x_row_of_w": ("s += gy[r * N + n] * w[n * K + k];", "s += gy[r * N + n] * w[(k * N + n) % (N * K)];"),
    "linear_grad_w_from_gx": ("s += gy[r * N + n] * x[r * K + k];", "s += gy[r * N + n] * gx[r * K + k];"),
}

PIN_CHECKS = [
    pins.test_golden_worked_bilinear,
    pins.test_golden_worked_two_level_fused,
    lambda o: pins.test_identity_at_pixel_centres(o, ((5, 7), (3, 11), (1, 1))),
    pins.test_constant_map,
    pins.test_linear_map_forward_and_backward,
    pins.test_backward_matches_central_differences,
    pins.test_fused_backward_matches_central_differences,
    pins.test_softmax_closed_forms,
    lambda o: pins.test_matches_torch_grid_sample(o, "ragged"),
]

DCN_PIN_CHECKS = [
    lambda o: dcn_pins.test_zero_offsets_are_a_depthwise_convolution((3, 3), (2, 2), (1, 1), (1, 1)),
    lambda o: dcn_pins.test_zero_offsets_are_a_depthwise_convolution((3, 3), (1, 1), (2, 2), (2, 2)),
    lambda o: dcn_pins.test_zero_offsets_are_a_depthwise_convolution((5, 3), (1, 2), (2, 1), (1, 1)),
    lambda o: dcn_pins.test_integer_and_half_pixel_offsets(),
    lambda o: dcn_pins.test_backward_finite_differences(),
    lambda o: dcn_pins.test_adjoint_identities(),
]


FP8_MUTATIONS = {
    "e4m3_exponent_bias_8": ("((unsigned)(E + 7) << 3)", "((unsigned)(E + 8) << 3)"),
    "e4m3_ties_away_from_zero": ("double r = nearbyint(a / quantum);", "double r = round(a / quantum);"),
    "e4m3_overflow_to_nan": ("    if (a >= 448.0)\n        return (unsigned char)(sign | 0x7E);",
                             "    if (a >= 448.0)\n        return (unsigned char)(sign | 0x7F);"),
    "e4m3_scale_127": ("amax > 0.0f ? amax / 448.0f : 1.0f", "amax > 0.0f ? amax / 127.0f : 1.0f"),
}

FP8_PIN_CHECKS = [
    lambda o: fp8_pins.test_spec_values(),
    lambda o: fp8_pins.test_every_code_round_trips(),
    lambda o: fp8_pins.test_ties_and_neighbours_match_brute_force(),
    lambda o: fp8_pins.test_matches_torch_float8_conversion(),
    lambda o: fp8_pins.test_quantiser_scale_and_error_bound(),
]

LINEAR_PIN_CHECKS = [
    linear_pins.test_golden_worked_linear,
    linear_pins.test_identity_and_zero_weights,
    linear_pins.test_adjoint_identities,
    linear_pins.test_query_head_column_order,
    linear_pins.test_query_head_backward_central_differences,
]


@contextlib.contextmanager
def _swapped(lib_path):
    oracle._load()
    saved = oracle._lib
    lib = ctypes.CDLL(lib_path)
    for name in ("msda_oracle_forward", "msda_oracle_backward", "msda_oracle_sampling_locations",
                 "msda_oracle_softmax", "msda_oracle_fused_chain", "msda_oracle_dcn_forward",
                 "msda_oracle_dcn_backward", "msda_oracle_linear", "msda_oracle_linear_backward",
                 "msda_oracle_e4m3_encode", "msda_oracle_e4m3_decode",
                 "msda_oracle_quantize_value_e4m3"):
        f, ref = getattr(lib, name), getattr(saved, name)
        f.argtypes, f.restype = ref.argtypes, ref.restype
    oracle._lib = lib
    saved_table, oracle._e4m3_table = oracle._e4m3_table, None
    try:
        yield
    finally:
        oracle._lib = saved
        oracle._e4m3_table = saved_table


ALL_MUTATIONS = {**MUTATIONS, **DCN_MUTATIONS, **LINEAR_MUTATIONS, **FP8_MUTATIONS}


@pytest.mark.parametrize("name", sorted(MUTATIONS) + sorted(DCN_MUTATIONS) + sorted(LINEAR_MUTATIONS)
                         + sorted(FP8_MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = ALL_MUTATIONS[name]
    checks = (PIN_CHECKS if name in MUTATIONS else
              DCN_PIN_CHECKS if name in DCN_MUTATIONS else
              LINEAR_PIN_CHECKS if name in LINEAR_MUTATIONS else FP8_PIN_CHECKS)
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    lib_path = str(tmp_path / "libmut.so")
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", lib_path,
                           str(mutated), "-lm"])
    failures = 0
    with _swapped(lib_path):
        for check in checks:
            try:
                check(oracle)
            except AssertionError:
                failures += 1
    assert failures > 0, f"mutation {name} passed every pin"
