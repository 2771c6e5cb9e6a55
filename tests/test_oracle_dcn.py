"""Pins of the oracle's DCNv3 core (discosf.com/news/5175395 §4.2: y(p0) =
sum_g sum_k w_g m_gk x_g(p0 + p_k + dp_gk); the core leaves w_g to a linear
layer).  With zero offsets the core is a depthwise convolution whose taps are
the masks, so torch's conv2d pins it; integer and half-pixel offsets reduce to
shifted and averaged inputs; the backward is pinned by finite differences and
by the two adjoint identities of a sum that is linear in x and in m."""
import numpy as np
import pytest
import torch

import oracle


def _x(N, H, W, G, C, seed=0):
    return np.random.default_rng(seed).normal(size=(N, H, W, G, C))


def _depthwise(x, taps, kernel, stride, pad, dil):
    """torch conv2d with one kh x kw filter per group, shared by its channels."""
    N, H, W, G, C = x.shape
    kh, kw = kernel
    xt = torch.from_numpy(x).permute(0, 3, 4, 1, 2).reshape(N, G * C, H, W)
    wt = torch.from_numpy(np.repeat(taps.reshape(G, 1, kh, kw), C, axis=0))  # [G*C, 1, kh, kw]
    y = torch.nn.functional.conv2d(xt, wt, stride=stride, padding=pad, dilation=dil, groups=G * C)
    Ho, Wo = y.shape[2], y.shape[3]
    return y.reshape(N, G, C, Ho, Wo).permute(0, 3, 4, 1, 2).numpy()


def test_centre_tap_is_identity():
    x = _x(2, 5, 7, 3, 8)
    Ho, Wo = oracle.dcn_output_size(5, 7, (3, 3), (1, 1), (1, 1))
    off = np.zeros((2, Ho, Wo, 3, 9, 2))
    m = np.zeros((2, Ho, Wo, 3, 9))
    m[..., 4] = 1.0
    assert np.array_equal(oracle.dcn_forward(x, off, m, (3, 3), (1, 1), (1, 1)), x)


@pytest.mark.parametrize("kernel,stride,pad,dil", [
    ((3, 3), (1, 1), (1, 1), (1, 1)),
    ((3, 3), (2, 2), (1, 1), (1, 1)),
    ((3, 3), (1, 1), (2, 2), (2, 2)),
    ((5, 3), (1, 2), (2, 1), (1, 1)),
    ((1, 1), (1, 1), (0, 0), (1, 1)),
])
def test_zero_offsets_are_a_depthwise_convolution(kernel, stride, pad, dil):
    x = _x(2, 9, 11, 2, 4, seed=1)
    K = kernel[0] * kernel[1]
    taps = np.random.default_rng(2).normal(size=(2, K))
    Ho, Wo = oracle.dcn_output_size(9, 11, kernel, stride, pad, dil)
    off = np.zeros((2, Ho, Wo, 2, K, 2))
    m = np.broadcast_to(taps[None, None, None], (2, Ho, Wo, 2, K)).copy()
    y = oracle.dcn_forward(x, off, m, kernel, stride, pad, dil)
    ref = _depthwise(x, taps, kernel, stride, pad, dil)
    assert y.shape == ref.shape
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_integer_and_half_pixel_offsets():
    """dx = +1 samples the next column, dx = +0.5 the mean of two columns,
    dy = -1 the row above (pixels outside the map read 0): the result is the
    plain convolution (no padding) of the array of what each padded tap reads."""
    x = _x(1, 6, 8, 2, 4, seed=3)
    kernel, stride, pad, dil = (3, 3), (1, 1), (1, 1), (1, 1)
    taps = np.random.default_rng(4).normal(size=(2, 9))
    Ho, Wo = oracle.dcn_output_size(6, 8, kernel, stride, pad, dil)
    m = np.broadcast_to(taps[None, None, None], (1, Ho, Wo, 2, 9)).copy()
    big = np.zeros((1, 6 + 4, 8 + 4, 2, 4))
    big[:, 2:-2, 2:-2] = x

    def val(r, c):  # x at rows r, columns c (arrays of the padded frame), 0 outside
        return big[:, 2 + r][:, :, 2 + c]

    rr, cc = np.arange(-1, 7), np.arange(-1, 9)  # padded frame: pixel -1 .. H, -1 .. W
    for dx, dy, reads in [
        (1.0, 0.0, val(rr, cc + 1)),
        (0.5, 0.0, 0.5 * (val(rr, cc) + val(rr, cc + 1))),
        (0.0, -1.0, val(rr - 1, cc)),
    ]:
        off = np.zeros((1, Ho, Wo, 2, 9, 2))
        off[..., 0], off[..., 1] = dx, dy
        y = oracle.dcn_forward(x, off, m, kernel, stride, pad, dil)
        np.testing.assert_allclose(y, _depthwise(reads, taps, kernel, stride, (0, 0), dil),
                                   rtol=1e-12, atol=1e-12)


def test_samples_beyond_one_pixel_are_dropped():
    x = _x(1, 4, 4, 1, 8, seed=5)
    off = np.zeros((1, 4, 4, 1, 1, 2))
    off[..., 0] = -1.0 - 0.0  # px = j - 1: column -1 exactly is outside for j = 0
    m = np.ones((1, 4, 4, 1, 1))
    y = oracle.dcn_forward(x, off, m, (1, 1))
    assert not y[:, :, 0].any()
    np.testing.assert_array_equal(y[:, :, 1:], x[:, :, :-1])


def test_backward_finite_differences():
    g = np.random.default_rng(6)
    kernel, stride, pad, dil = (3, 3), (1, 1), (1, 1), (1, 1)
    x = g.normal(size=(1, 4, 5, 2, 3))
    Ho, Wo = oracle.dcn_output_size(4, 5, kernel, stride, pad, dil)
    off = g.uniform(-1.3, 1.3, size=(1, Ho, Wo, 2, 9, 2))
    m = g.normal(size=(1, Ho, Wo, 2, 9))
    gy = g.normal(size=(1, Ho, Wo, 2, 3))
    gx, goff, gm = oracle.dcn_backward(x, off, m, gy, kernel, stride, pad, dil)
    f = lambda xx, oo, mm: float((oracle.dcn_forward(xx, oo, mm, kernel, stride, pad, dil) * gy).sum())
    h = 1e-6
    for idx in [(0, 1, 2, 0, 3, 0), (0, 0, 0, 1, 0, 1), (0, 3, 4, 1, 8, 0), (0, 2, 1, 0, 5, 1)]:
        op, om = off.copy(), off.copy()
        op[idx] += h
        om[idx] -= h
        assert abs((f(x, op, m) - f(x, om, m)) / (2 * h) - goff[idx]) < 1e-6
    for idx in [(0, 1, 2, 0, 3), (0, 3, 4, 1, 8)]:
        mp = m.copy()
        mp[idx] += 1.0
        assert abs(f(x, off, mp) - f(x, off, m) - gm[idx]) < 1e-9  # linear in m
    for idx in [(0, 1, 2, 0, 1), (0, 3, 4, 1, 2), (0, 0, 0, 0, 0)]:
        xp = x.copy()
        xp[idx] += 1.0
        assert abs(f(xp, off, m) - f(x, off, m) - gx[idx]) < 1e-9  # linear in x


def test_adjoint_identities():
    """<grad_x, x> = <grad_y, y> = <grad_mask, mask>: the sum is linear in x
    and in m separately."""
    g = np.random.default_rng(7)
    kernel, stride, pad, dil = (3, 3), (2, 2), (1, 1), (1, 1)
    x = g.normal(size=(2, 7, 9, 3, 4))
    Ho, Wo = oracle.dcn_output_size(7, 9, kernel, stride, pad, dil)
    off = g.normal(size=(2, Ho, Wo, 3, 9, 2)) * 1.5
    m = g.normal(size=(2, Ho, Wo, 3, 9))
    gy = g.normal(size=(2, Ho, Wo, 3, 4))
    y = oracle.dcn_forward(x, off, m, kernel, stride, pad, dil)
    gx, _, gm = oracle.dcn_backward(x, off, m, gy, kernel, stride, pad, dil)
    rhs = float((gy * y).sum())
    assert abs(float((gx * x).sum()) - rhs) < 1e-9 * max(1.0, abs(rhs))
    assert abs(float((gm * m).sum()) - rhs) < 1e-9 * max(1.0, abs(rhs))


def test_matches_the_attention_oracle_on_one_level():
    """The same sampling written through the attention core: one level, heads
    = groups, the location of each point given in normalized units."""
    g = np.random.default_rng(8)
    kernel, stride, pad, dil = (3, 3), (1, 1), (1, 1), (1, 1)
    N, H, W, G, C = 1, 6, 7, 2, 8
    x = g.normal(size=(N, H, W, G, C))
    Ho, Wo = oracle.dcn_output_size(H, W, kernel, stride, pad, dil)
    off = g.normal(size=(N, Ho, Wo, G, 9, 2))
    m = g.normal(size=(N, Ho, Wo, G, 9))
    y = oracle.dcn_forward(x, off, m, kernel, stride, pad, dil)
    ii, jj = np.meshgrid(np.arange(Ho), np.arange(Wo), indexing="ij")
    r, c = np.arange(9) // 3, np.arange(9) % 3
    px = (jj[:, :, None, None] - 1 + c[None, None, None, :]) + off[0, ..., 0]
    py = (ii[:, :, None, None] - 1 + r[None, None, None, :]) + off[0, ..., 1]
    loc = np.stack([(px + 0.5) / W, (py + 0.5) / H], -1).reshape(N, Ho * Wo, G, 1, 9, 2)
    out = oracle.forward(x.reshape(N, H * W, G, C), np.array([[H, W]]), np.array([0]), loc,
                         m.reshape(N, Ho * Wo, G, 1, 9))
    np.testing.assert_allclose(out.reshape(y.shape), y, rtol=1e-9, atol=1e-9)
