"""Property checks of the oracle over generated shapes (hypothesis,
derandomized so the suite is reproducible): the core sum is linear in the
value map and in the attention weights, so its backward must satisfy
<grad_value, value> = <grad_out, out> = <grad_attn, attn> at any shape; the
fused chain's softmax rows sum to 1 and its logit gradients sum to 0 per row
(the softmax Jacobian annihilates constants); the DCNv3 core obeys the same
two identities."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    L = draw(st.integers(1, 3))
    levels = [(draw(st.integers(1, 6)), draw(st.integers(1, 6))) for _ in range(L)]
    Q = draw(st.integers(1, 5))
    M = draw(st.integers(1, 3))
    D = draw(st.sampled_from([1, 2, 4]))
    K = draw(st.integers(1, 3))
    seed = draw(st.integers(0, 2**31 - 1))
    return B, levels, Q, M, D, K, seed


def _inputs(B, levels, Q, M, D, K, seed):
    g = np.random.default_rng(seed)
    L = len(levels)
    S = sum(h * w for h, w in levels)
    shapes = np.array(levels, dtype=np.int64)
    starts = np.concatenate([[0], np.cumsum([h * w for h, w in levels])[:-1]]).astype(np.int64)
    value = g.normal(size=(B, S, M, D))
    loc = g.uniform(-0.3, 1.3, size=(B, Q, M, L, K, 2))
    attn = g.normal(size=(B, Q, M, L, K))
    gout = g.normal(size=(B, Q, M, D))
    return shapes, starts, value, loc, attn, gout


@SETTINGS
@given(problems())
def test_adjoint_identities(p):
    shapes, starts, value, loc, attn, gout = _inputs(*p)
    out = oracle.forward(value, shapes, starts, loc, attn)
    gv, gl, ga = oracle.backward(value, shapes, starts, loc, attn, gout)
    rhs = float((gout * out).sum())
    scale = max(1.0, float(np.abs(gout).sum() * np.abs(value).max() * np.abs(attn).max()))
    assert abs(float((gv * value).sum()) - rhs) <= 1e-12 * scale
    assert abs(float((ga * attn).sum()) - rhs) <= 1e-12 * scale
    assert gl.shape == loc.shape and np.isfinite(gl).all()


@SETTINGS
@given(problems())
def test_fused_softmax_rows(p):
    B, levels, Q, M, D, K, seed = p
    shapes, starts, value, _, _, gout = _inputs(*p)
    g = np.random.default_rng(seed + 1)
    L = len(levels)
    ref = g.uniform(0, 1, size=(B, Q, 2))
    off = g.normal(size=(B, Q, M, L, K, 2))
    logits = 3.0 * g.normal(size=(B, Q, M, L * K))
    out, a, _ = oracle.fused_forward(value, shapes, starts, ref, off, logits)
    np.testing.assert_allclose(a.reshape(B, Q, M, -1).sum(-1), 1.0, rtol=1e-12)
    _, _, _, glog = oracle.fused_backward(value, shapes, starts, ref, off, logits, gout)
    row = np.abs(glog).sum(-1) + 1e-300
    assert np.all(np.abs(glog.sum(-1)) <= 1e-12 * np.maximum(row, 1.0))


@SETTINGS
@given(st.integers(1, 2), st.integers(1, 7), st.integers(1, 7), st.integers(1, 3),
       st.sampled_from([1, 2]), st.sampled_from([(1, 1), (2, 2), (3, 3), (3, 2)]),
       st.integers(1, 2), st.integers(0, 2), st.integers(0, 2**31 - 1))
def test_dcn_adjoint_identities(N, H, W, G, C, kernel, stride, pad, seed):
    g = np.random.default_rng(seed)
    Ho, Wo = oracle.dcn_output_size(H, W, kernel, (stride, stride), (pad, pad), (1, 1))
    if Ho < 1 or Wo < 1:
        return
    K = kernel[0] * kernel[1]
    x = g.normal(size=(N, H, W, G, C))
    off = 1.5 * g.normal(size=(N, Ho, Wo, G, K, 2))
    m = g.normal(size=(N, Ho, Wo, G, K))
    gy = g.normal(size=(N, Ho, Wo, G, C))
    geo = dict(kernel=kernel, stride=(stride, stride), pad=(pad, pad), dil=(1, 1))
    y = oracle.dcn_forward(x, off, m, **geo)
    gx, _, gm = oracle.dcn_backward(x, off, m, gy, **geo)
    rhs = float((gy * y).sum())
    scale = max(1.0, float(np.abs(gy).sum() * np.abs(x).max() * np.abs(m).max()))
    assert abs(float((gx * x).sum()) - rhs) <= 1e-12 * scale
    assert abs(float((gm * m).sum()) - rhs) <= 1e-12 * scale
