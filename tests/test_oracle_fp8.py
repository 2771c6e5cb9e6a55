"""Pins of the oracle's FP8 (E4M3) value storage (CPU only).

The format is the E4M3 encoding of the OCP 8-bit floating-point
specification: sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent
field 0 holds the subnormals m/8 * 2^-6, S.1111.111 is NaN, no infinities,
largest finite magnitude 448.  The pins check the oracle's codec against
values the definition fixes, against a brute-force nearest-value search over
all 256 codes, and against torch's own float8_e4m3fn conversion (a library
routine that shares nothing with the oracle), then the quantiser's scale and
error bounds.
"""
import numpy as np
import pytest
import torch

import oracle

# (code, value) pairs the definition fixes
SPEC = [
    (0x00, 0.0), (0x80, -0.0), (0x38, 1.0), (0xB8, -1.0), (0x40, 2.0), (0x30, 0.5),
    (0x39, 1.125), (0x3F, 1.875), (0x7E, 448.0), (0xFE, -448.0), (0x77, 240.0),
    (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x04, 2.0 ** -7),
]


def _brute_encode(x: float) -> int:
    """The code of the finite value nearest to x, ties to the even mantissa
    (code bit 0), clipped to +-448, by search over every code."""
    if abs(x) >= 448.0:
        return 0xFE if x < 0 else 0x7E
    table = oracle.e4m3_decode(np.arange(256))
    best, best_d = None, None
    for c in range(256):
        v = table[c]
        if np.isnan(v) or (np.signbit(v) != np.signbit(x)):
            continue
        d = abs(v - x)
        if best is None or d < best_d or (d == best_d and (c & 1) == 0 and (best & 1) == 1):
            best, best_d = c, d
    return best


def test_spec_values():
    for code, value in SPEC:
        got = oracle.e4m3_decode(code)
        assert got == value and np.signbit(got) == np.signbit(value), hex(code)
        assert int(oracle.e4m3_encode(np.float32(value))) == code, hex(code)
    assert np.isnan(oracle.e4m3_decode(0x7F)) and np.isnan(oracle.e4m3_decode(0xFF))


def test_every_code_round_trips():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if np.isnan(v):
            continue
        assert int(oracle.e4m3_encode(np.float32(v))) == c, hex(c)


def test_ties_and_neighbours_match_brute_force():
    """Every midpoint between consecutive magnitudes (a tie), and points a
    little to either side, encode as the brute-force nearest search does."""
    mags = sorted({abs(oracle.e4m3_decode(c)) for c in range(128) if not np.isnan(oracle.e4m3_decode(c))})
    xs = []
    for lo, hi in zip(mags[:-1], mags[1:]):
        mid = (lo + hi) / 2
        xs += [mid, np.nextafter(np.float32(mid), np.float32(0)), np.nextafter(np.float32(mid), np.float32(1e9))]
    xs += [449.0, 463.9, 464.0, 1e6]
    for x in xs:
        for sx in (np.float32(x), np.float32(-x)):
            assert int(oracle.e4m3_encode(sx)) == _brute_encode(float(sx)), float(sx)


def test_matches_torch_float8_conversion():
    """torch's float8_e4m3fn conversion (round to nearest even) gives the same
    codes for values inside the finite range."""
    rng = np.random.default_rng(20261203)
    x = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 100, 4000), rng.uniform(-460, 460, 2000),
                        rng.normal(0, 2.0 ** -7, 2000)]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:10]


def test_quantiser_scale_and_error_bound():
    rng = np.random.default_rng(7)
    v = rng.normal(0, 1, (2, 50, 3, 16)).astype(np.float32)
    v[1, :, 2, :] = 0.0                             # an all-zero (batch, head)
    v[0, 17, 1, 5] = -9.5                           # its head's absmax, negative
    q, scale = oracle.quantize_value_e4m3(v)
    assert q.dtype == np.uint8 and scale.shape == (2, 3)
    amax = np.abs(v).max(axis=(1, 3))
    want_scale = np.where(amax > 0, (amax / np.float32(448)).astype(np.float32), np.float32(1))
    assert np.array_equal(scale, want_scale)
    assert q[0, 17, 1, 5] == 0xFE                   # -amax lands on -448
    assert not q[1, :, 2, :].any()
    deq = oracle.dequantize_value_e4m3(q, scale)
    # within half a quantum of x = value / scale: 2^-4 of |x| for normals,
    # 2^-10 absolute in the subnormal range, in units of the scale
    x = v.astype(np.float64) / scale[:, None, :, None]
    err = np.abs(deq / scale[:, None, :, None] - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
    assert (err <= bound).all()


@pytest.mark.parametrize("seed", [1, 2])
def test_quantiser_codes_follow_the_codec(seed):
    """The quantiser's codes are the codec's on value / scale in float32."""
    rng = np.random.default_rng(seed)
    v = rng.normal(0, 3, (1, 40, 2, 8)).astype(np.float32)
    q, scale = oracle.quantize_value_e4m3(v)
    x = (v / scale[:, None, :, None]).astype(np.float32)
    assert np.array_equal(q, oracle.e4m3_encode(x))
