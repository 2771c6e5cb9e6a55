"""Pins of the oracle's INT8 value storage (symmetric, one absmax scale per
(batch, head), round half to even), against values fixed by the definition,
closed forms, invariants and numpy's own rounding.  The INT8 idea comes from
the quantisation note of the x-humanoid.csdn.net MSDA explainer (§4); the
scheme is the reading recorded in the oracle's header."""
import numpy as np
import pytest

import oracle
from scale_deformable_attention_msdeformattn_b200 import workloads as wl


def test_rounding_is_half_to_even():
    # amax = 127 makes the scale exactly 1, so q is value rounded to an integer
    v = np.array([2.5, 3.5, -2.5, -0.5, 127.0, 0.0, 1.49, -127.0, 0.5, 1.5, -1.5, 126.5],
                 np.float32).reshape(1, 1, 1, 12)
    q, scale = oracle.quantize_value_s8(v)
    assert scale.tolist() == [[1.0]]
    assert q.ravel().tolist() == [2, 4, -2, 0, 127, 0, 1, -127, 0, 2, -2, 126]


def test_exact_grid_round_trips():
    """Values k * 2^-3 with max |k| = 127 have scale 2^-3 exactly and q = k."""
    g = np.random.default_rng(1)
    k = g.integers(-127, 128, size=(2, 9, 3, 16))
    k[:, 0, :, 0] = 127
    v = (k * 0.125).astype(np.float32)
    q, scale = oracle.quantize_value_s8(v)
    assert np.all(scale == np.float32(0.125))
    assert np.array_equal(q.astype(np.int64), k)
    assert np.array_equal(oracle.dequantize_value_s8(q, scale), k * 0.125)


def test_zero_head_has_unit_scale():
    v = np.zeros((1, 5, 2, 8), np.float32)
    v[0, :, 1, :] = np.linspace(-1, 1, 40, dtype=np.float32).reshape(5, 8)
    q, scale = oracle.quantize_value_s8(v)
    assert scale[0, 0] == 1.0 and not q[0, :, 0, :].any()
    assert scale[0, 1] == np.float32(1.0) / np.float32(127.0)


def test_heads_are_independent_and_scale_with_powers_of_two():
    g = np.random.default_rng(2)
    v = g.normal(size=(2, 11, 4, 8)).astype(np.float32)
    q, scale = oracle.quantize_value_s8(v)
    v2 = v.copy()
    v2[1, :, 2, :] *= 4.0
    q2, scale2 = oracle.quantize_value_s8(v2)
    assert scale2[1, 2] == 4.0 * scale[1, 2]
    assert np.array_equal(q2, q)
    mask = np.ones_like(scale, bool)
    mask[1, 2] = False
    assert np.array_equal(scale2[mask], scale[mask])


def test_error_is_at_most_half_a_step():
    g = np.random.default_rng(3)
    v = g.normal(size=(2, 50, 3, 16)).astype(np.float32) * np.float32(3.0)
    q, scale = oracle.quantize_value_s8(v)
    err = np.abs(oracle.dequantize_value_s8(q, scale) - v.astype(np.float64))
    step = scale.astype(np.float64)[:, None, :, None]
    assert np.all(err <= 0.5000001 * step)
    assert np.abs(q.astype(np.int64)).max() == 127


def test_matches_numpy_float32_scale_and_rint():
    """The same scheme written with numpy's own float32 division and rint."""
    g = np.random.default_rng(4)
    v = (g.normal(size=(3, 40, 2, 32)) * g.uniform(0.1, 10.0, size=(3, 1, 2, 1))).astype(np.float32)
    q, scale = oracle.quantize_value_s8(v)
    amax = np.abs(v).max(axis=(1, 3))
    ref_scale = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(scale, ref_scale)
    ref_q = np.clip(np.rint(v / ref_scale[:, None, :, None]), -127, 127).astype(np.int8)
    assert np.array_equal(q, ref_q)


def test_bfloat16_source_is_widened_exactly():
    x = wl.normal(77, 1, 2 * 6 * 2 * 8).reshape(2, 6, 2, 8)
    bits = wl.to_bf16_bits(x)
    q1, s1 = oracle.quantize_value_s8(bits)
    q2, s2 = oracle.quantize_value_s8(wl.bf16_bits_to_f64(bits).astype(np.float32))
    assert np.array_equal(q1, q2) and np.array_equal(s1, s2)


@pytest.mark.parametrize("bad", ["amax_over_all_heads", "truncate"])
def test_pins_catch_planted_mistakes(bad):
    """Two plausible mistakes, planted in a copy of the scheme, fail the pins
    above (the pins are not tautologies)."""
    v = np.array([2.5, 3.5, -2.5, -0.5, 127.0, 0.0, 1.49, -127.0], np.float32).reshape(1, 1, 1, 8)
    v2 = np.concatenate([v, v * 0.5], axis=2)  # two heads

    def planted(x):
        if bad == "amax_over_all_heads":
            amax = np.abs(x).max()
            sc = np.full((x.shape[0], x.shape[2]), amax / np.float32(127.0), np.float32)
        else:
            sc = np.abs(x).max(axis=(1, 3)) / np.float32(127.0)
        r = x / sc[:, None, :, None]
        r = np.trunc(r) if bad == "truncate" else np.rint(r)
        return np.clip(r, -127, 127).astype(np.int8), sc.astype(np.float32)

    q, s = planted(v2)
    qo, so = oracle.quantize_value_s8(v2)
    assert not (np.array_equal(q, qo) and np.array_equal(s, so))
