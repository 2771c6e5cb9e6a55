"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

None of these compares the oracle with itself: each check is a hand-worked
example (tests/golden), a closed form, an identity that holds for every input,
a library routine the pages name (torch grid_sample, cf-1.com/news/4799680
§5.3), or finite differences of the forward.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from scale_deformable_attention_msdeformattn_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _starts(shapes):
    return wl.level_start_index([tuple(s) for s in shapes])


def _random_problem(rng, B=2, levels=((5, 7), (3, 4)), Q=3, M=2, D=3, K=2, margin=True):
    """fp64 inputs whose samples keep 0.1 px away from every cell edge, so
    that finite differences stay inside one bilinear cell."""
    L = len(levels)
    shapes = np.array(levels, np.int64)
    S = int((shapes[:, 0] * shapes[:, 1]).sum())
    value = rng.standard_normal((B, S, M, D))
    loc = np.empty((B, Q, M, L, K, 2))
    for l, (H, W) in enumerate(levels):
        # integer cell in [-1, W-1] so that border cells (partly outside) occur
        cx = rng.integers(-1, W, size=(B, Q, M, K))
        cy = rng.integers(-1, H, size=(B, Q, M, K))
        fx = rng.uniform(0.1, 0.9, size=(B, Q, M, K))
        fy = rng.uniform(0.1, 0.9, size=(B, Q, M, K))
        loc[:, :, :, l, :, 0] = (cx + fx + 0.5) / W
        loc[:, :, :, l, :, 1] = (cy + fy + 0.5) / H
    attn = rng.uniform(0.1, 1.0, size=(B, Q, M, L, K))
    g = rng.standard_normal((B, Q, M, D))
    return value, shapes, _starts(levels), loc, attn, g


# ---------------------------------------------------------------- golden ---

def test_golden_worked_bilinear(oracle_mod):
    fx = json.load(open(os.path.join(GOLDEN, "worked_bilinear_2x3.json")))
    shapes = np.array(fx["spatial_shapes"], np.int64)
    value = np.array(fx["value"], np.float64).reshape(1, 6, 1, 1)
    loc = np.array(fx["sampling_locations"], np.float64).reshape(1, 5, 1, 1, 1, 2)
    attn = np.ones((1, 5, 1, 1, 1))
    out = oracle_mod.forward(value, shapes, [0], loc, attn)
    np.testing.assert_allclose(out.ravel(), fx["expected_out"], rtol=0, atol=1e-14)
    gv, gl, ga = oracle_mod.backward(value, shapes, [0], loc, attn, np.ones((1, 5, 1, 1)))
    np.testing.assert_allclose(gl.reshape(5, 2), fx["expected_grad_loc"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(ga.ravel(), fx["expected_grad_attn"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(gv.ravel(), fx["expected_grad_value"], rtol=0, atol=1e-14)


def test_golden_worked_two_level_fused(oracle_mod):
    fx = json.load(open(os.path.join(GOLDEN, "worked_two_level_fused.json")))
    shapes = np.array(fx["spatial_shapes"], np.int64)
    starts = _starts(shapes)
    value = np.array(fx["value"], np.float64).reshape(1, 6, 1, 1)
    ref = np.array(fx["reference_points"], np.float64).reshape(1, 1, 2)
    off = np.array(fx["sampling_offsets"], np.float64).reshape(1, 1, 1, 2, 1, 2)
    logits = np.array(fx["attention_logits"], np.float64).reshape(1, 1, 1, 2)
    out, a, loc = oracle_mod.fused_forward(value, shapes, starts, ref, off, logits)
    assert abs(out.item() - fx["expected_out"]) < 1e-14
    np.testing.assert_allclose(a.ravel(), fx["expected_attention_weights"], atol=1e-15)
    gv, gref, goff, glog = oracle_mod.fused_backward(value, shapes, starts, ref, off, logits,
                                                     np.ones((1, 1, 1, 1)))
    np.testing.assert_allclose(glog.ravel(), fx["expected_grad_logits"], atol=1e-13)
    np.testing.assert_allclose(goff.reshape(2, 2), fx["expected_grad_offsets"], atol=1e-13)
    np.testing.assert_allclose(gref.ravel(), fx["expected_grad_ref"], atol=1e-13)
    np.testing.assert_allclose(gv.ravel(), fx["expected_grad_value"], atol=1e-14)


# ------------------------------------------------------------ closed forms ---

@pytest.mark.parametrize("levels", [((8, 8), (4, 4)), ((5, 7), (3, 11), (1, 1))])
def test_identity_at_pixel_centres(oracle_mod, levels):
    """Zero offset at a pixel centre returns that pixel's value exactly
    (discosf.com/news/5175395 §3.1: zero offsets sample the reference point;
    pixel centres from cf-1.com/news/4799680 §3.2)."""
    rng = np.random.default_rng(1)
    B, Q, M, D, K = 2, 5, 3, 4, 3
    L = len(levels)
    shapes = np.array(levels, np.int64)
    starts = _starts(levels)
    S = int((shapes[:, 0] * shapes[:, 1]).sum())
    # every element distinct, so any index slip (level start, row/column,
    # head, channel, batch) changes the answer
    value = np.arange(B * S * M * D, dtype=np.float64).reshape(B, S, M, D) * 0.5 + 1.0
    loc = np.empty((B, Q, M, L, K, 2))
    expect = np.zeros((B, Q, M, D))
    attn = rng.uniform(0.0, 1.0, size=(B, Q, M, L, K))
    for b in range(B):
        for q in range(Q):
            for m in range(M):
                for l, (H, W) in enumerate(levels):
                    for k in range(K):
                        i, j = rng.integers(0, H), rng.integers(0, W)
                        loc[b, q, m, l, k] = ((j + 0.5) / W, (i + 0.5) / H)
                        expect[b, q, m] += attn[b, q, m, l, k] * value[b, starts[l] + i * W + j, m]
    out = oracle_mod.forward(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out, expect, rtol=1e-13, atol=0)


def test_constant_map(oracle_mod):
    """value = c everywhere, all corners inside, sum A = 1 -> out = c and
    grad_loc = 0 (cf-1.com/news/4799680 §3.1: the weights sum to 1)."""
    rng = np.random.default_rng(2)
    levels = ((6, 9), (3, 5))
    shapes = np.array(levels, np.int64)
    B, Q, M, D, K = 1, 7, 2, 5, 4
    L = 2
    S = 6 * 9 + 3 * 5
    c = rng.standard_normal((M, D))
    value = np.broadcast_to(c, (B, S, M, D)).copy()
    loc = np.empty((B, Q, M, L, K, 2))
    for l, (H, W) in enumerate(levels):
        x = rng.uniform(0.0, W - 1, size=(B, Q, M, K))
        y = rng.uniform(0.0, H - 1, size=(B, Q, M, K))
        loc[..., l, :, 0] = (x + 0.5) / W
        loc[..., l, :, 1] = (y + 0.5) / H
    attn = rng.uniform(0.1, 1, size=(B, Q, M, L, K))
    attn /= attn.sum(axis=(3, 4), keepdims=True)
    out = oracle_mod.forward(value, shapes, _starts(levels), loc, attn)
    np.testing.assert_allclose(out, np.broadcast_to(c, out.shape), rtol=1e-13, atol=1e-13)
    g = rng.standard_normal((B, Q, M, D))
    _, gl, _ = oracle_mod.backward(value, shapes, _starts(levels), loc, attn, g)
    assert np.abs(gl).max() < 1e-12


def test_linear_map_forward_and_backward(oracle_mod):
    """v(y, x) = a + b x + c y is reproduced exactly by bilinear sampling, and
    the location gradients are W*A*<g,b>, H*A*<g,c> (the pixel coordinate is
    loc*W - 0.5: cf-1.com/news/4799680 §5.3, grid_sample align_corners=False)."""
    rng = np.random.default_rng(3)
    levels = ((5, 11), (7, 3))
    shapes = np.array(levels, np.int64)
    starts = _starts(levels)
    B, Q, M, D, K, L = 2, 6, 2, 3, 3, 2
    S = 5 * 11 + 7 * 3
    a = rng.standard_normal((L, M, D))
    bx = rng.standard_normal((L, M, D))
    cy = rng.standard_normal((L, M, D))
    value = np.empty((B, S, M, D))
    for l, (H, W) in enumerate(levels):
        for i in range(H):
            for j in range(W):
                value[:, starts[l] + i * W + j] = a[l] + bx[l] * j + cy[l] * i
    loc = np.empty((B, Q, M, L, K, 2))
    px = np.empty((B, Q, M, L, K, 2))
    for l, (H, W) in enumerate(levels):
        x = rng.uniform(0.0, W - 1, size=(B, Q, M, K))
        y = rng.uniform(0.0, H - 1, size=(B, Q, M, K))
        px[..., l, :, 0], px[..., l, :, 1] = x, y
        loc[..., l, :, 0] = (x + 0.5) / W
        loc[..., l, :, 1] = (y + 0.5) / H
    attn = rng.uniform(0.1, 1, size=(B, Q, M, L, K))
    g = rng.standard_normal((B, Q, M, D))
    expect = np.zeros((B, Q, M, D))
    egl = np.zeros((B, Q, M, L, K, 2))
    ega = np.zeros((B, Q, M, L, K))
    for l, (H, W) in enumerate(levels):
        for k in range(K):
            samp = (a[l][None, None] + bx[l][None, None] * px[:, :, :, l, k, 0, None]
                    + cy[l][None, None] * px[:, :, :, l, k, 1, None])
            expect += attn[:, :, :, l, k, None] * samp
            ega[:, :, :, l, k] = (g * samp).sum(-1)
            egl[:, :, :, l, k, 0] = W * attn[:, :, :, l, k] * (g * bx[l][None, None]).sum(-1)
            egl[:, :, :, l, k, 1] = H * attn[:, :, :, l, k] * (g * cy[l][None, None]).sum(-1)
    out = oracle_mod.forward(value, shapes, starts, loc, attn)
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-12)
    _, gl, ga = oracle_mod.backward(value, shapes, starts, loc, attn, g)
    np.testing.assert_allclose(ga, ega, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gl, egl, rtol=1e-11, atol=1e-11)


def test_coincident_points_equal_single_sample(oracle_mod):
    """K identical points with weights A_k equal one point with weight sum A_k."""
    rng = np.random.default_rng(4)
    value, shapes, starts, loc, attn, g = _random_problem(rng, K=4)
    loc_same = loc.copy()
    loc_same[..., :, :] = loc[..., 0:1, :]
    out_k = oracle_mod.forward(value, shapes, starts, loc_same, attn)
    one_loc = loc[..., 0:1, :]
    one_attn = attn.sum(-1, keepdims=True)
    out_1 = oracle_mod.forward(value, shapes, starts, np.ascontiguousarray(one_loc), one_attn)
    np.testing.assert_allclose(out_k, out_1, rtol=1e-13, atol=1e-13)


def test_out_of_range_sample_is_zero(oracle_mod):
    """A sample with x <= -1, x >= W, y <= -1 or y >= H contributes nothing and
    has zero gradients (discosf.com/news/5175395 §2.2: masked to zero)."""
    rng = np.random.default_rng(5)
    value, shapes, starts, loc, attn, g = _random_problem(rng)
    W0, H0 = shapes[0, 1], shapes[0, 0]
    far = [(-1.0 / W0 * 0.6, 0.5), (1.0 + 0.51 / W0, 0.5), (0.5, -0.6 / H0), (0.5, 1.0 + 0.6 / H0),
           (-3.0, -3.0)]
    out_ref = oracle_mod.forward(value, shapes, starts, loc, attn)
    for (x, y) in far:
        loc2 = loc.copy()
        loc2[0, 0, 0, 0, 0] = (x, y)
        # the sample's own contribution, computed by moving it out of range
        out2 = oracle_mod.forward(value, shapes, starts, loc2, attn)
        attn_z = attn.copy()
        attn_z[0, 0, 0, 0, 0] = 0.0
        out_z = oracle_mod.forward(value, shapes, starts, loc, attn_z)
        np.testing.assert_allclose(out2, out_z, rtol=1e-13, atol=1e-13)
        _, gl, ga = oracle_mod.backward(value, shapes, starts, loc2, attn, g)
        assert gl[0, 0, 0, 0, 0].tolist() == [0.0, 0.0] and ga[0, 0, 0, 0, 0] == 0.0
    assert np.abs(out_ref).max() > 0


def test_permuting_points_with_weights(oracle_mod):
    rng = np.random.default_rng(6)
    value, shapes, starts, loc, attn, g = _random_problem(rng, K=3)
    perm = [2, 0, 1]
    out = oracle_mod.forward(value, shapes, starts, loc, attn)
    out_p = oracle_mod.forward(value, shapes, starts, np.ascontiguousarray(loc[..., perm, :]),
                               np.ascontiguousarray(attn[..., perm]))
    np.testing.assert_allclose(out, out_p, rtol=1e-13, atol=1e-13)


def test_linearity_in_value_and_weights(oracle_mod):
    rng = np.random.default_rng(7)
    value, shapes, starts, loc, attn, g = _random_problem(rng)
    v2 = rng.standard_normal(value.shape)
    a2 = rng.uniform(0, 1, attn.shape)
    f = lambda v, a: oracle_mod.forward(v, shapes, starts, loc, a)
    np.testing.assert_allclose(f(2 * value - 3 * v2, attn), 2 * f(value, attn) - 3 * f(v2, attn),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(value, attn + a2), f(value, attn) + f(value, a2),
                               rtol=1e-12, atol=1e-12)


def test_adjoint_identities(oracle_mod):
    """out is linear in value and in A, so <grad_value, value> = <g, out> and
    <grad_attn, A> = <g, out> (holds with out-of-range samples too)."""
    w = wl.custom("adj", 2, [(9, 13), (5, 7), (2, 3)], 40, 3, 8, 3, offset_sigma=3.0)
    x = wl.generate(w)
    v, g = x.value_f64(), x.grad_output_f64()
    out = oracle_mod.forward(v, x.spatial_shapes, x.level_start_index, x.sampling_locations,
                             x.attention_weights)
    gv, gl, ga = oracle_mod.backward(v, x.spatial_shapes, x.level_start_index,
                                     x.sampling_locations, x.attention_weights, g)
    rhs = float((g * out).sum())
    assert abs(float((gv * v).sum()) - rhs) < 1e-10 * max(1.0, abs(rhs))
    assert abs(float((ga * x.attention_weights).sum()) - rhs) < 1e-10 * max(1.0, abs(rhs))


# --------------------------------------------------------- finite differences

def _fd(f, x, h):
    gr = np.empty_like(x)
    flat = x.reshape(-1)
    gflat = gr.reshape(-1)
    for i in range(flat.size):
        old = flat[i]
        flat[i] = old + h
        fp = f()
        flat[i] = old - h
        fm = f()
        flat[i] = old
        gflat[i] = (fp - fm) / (2 * h)
    return gr


def test_backward_matches_central_differences(oracle_mod):
    """Bilinear sampling is differentiable in the coordinates
    (discosf.com/news/5175395 §2.1); inside one cell it is linear in each
    coordinate, so central differences are exact up to rounding."""
    rng = np.random.default_rng(8)
    value, shapes, starts, loc, attn, g = _random_problem(rng)
    f = lambda: float((g * oracle_mod.forward(value, shapes, starts, loc, attn)).sum())
    gv, gl, ga = oracle_mod.backward(value, shapes, starts, loc, attn, g)
    np.testing.assert_allclose(_fd(f, loc, 1e-7), gl, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(_fd(f, attn, 1e-6), ga, rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(_fd(f, value, 1e-6), gv, rtol=1e-7, atol=1e-8)


def test_fused_backward_matches_central_differences(oracle_mod):
    """Chain rule through loc = ref + off/(W,H) and the softmax over L*K
    (cf-1.com/news/4799680 §3.2)."""
    rng = np.random.default_rng(9)
    value, shapes, starts, loc, attn, g = _random_problem(rng, B=1, Q=2, M=2, D=2, K=2)
    B, Q, M, L, K, _ = loc.shape
    # ref at a fixed point; offsets chosen so that ref + off/(W,H) == loc
    ref = rng.uniform(0.2, 0.8, size=(B, Q, 2))
    W = shapes[:, 1].astype(float)[None, None, None, :, None]
    H = shapes[:, 0].astype(float)[None, None, None, :, None]
    off = np.empty_like(loc)
    off[..., 0] = (loc[..., 0] - ref[:, :, None, None, None, 0]) * W
    off[..., 1] = (loc[..., 1] - ref[:, :, None, None, None, 1]) * H
    logits = rng.standard_normal((B, Q, M, L * K))
    f = lambda: float((g * oracle_mod.fused_forward(value, shapes, starts, ref, off, logits)[0]).sum())
    gv, gref, goff, glog = oracle_mod.fused_backward(value, shapes, starts, ref, off, logits, g)
    np.testing.assert_allclose(_fd(f, off, 1e-6), goff, rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(_fd(f, ref, 1e-8), gref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(_fd(f, logits, 1e-5), glog, rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(_fd(f, value, 1e-6), gv, rtol=1e-7, atol=1e-8)


# ---------------------------------------------------------------- softmax ---

def test_softmax_closed_forms(oracle_mod):
    """Rows sum to 1 (cf-1.com/news/4799680 §3.1); shift invariance; two
    logits give the logistic function; equal logits give 1/(L*K)."""
    rng = np.random.default_rng(10)
    z = rng.standard_normal((2, 3, 4, 6)) * 5
    a = oracle_mod.softmax(z, 2, 3).reshape(z.shape)
    np.testing.assert_allclose(a.sum(-1), 1.0, atol=1e-14)
    a2 = oracle_mod.softmax(z + 100.0, 2, 3).reshape(z.shape)
    np.testing.assert_allclose(a, a2, rtol=1e-12)
    z2 = rng.standard_normal((1, 1, 5, 2))
    a3 = oracle_mod.softmax(z2, 1, 2).reshape(z2.shape)
    np.testing.assert_allclose(a3[..., 0], 1.0 / (1.0 + np.exp(z2[..., 1] - z2[..., 0])), rtol=1e-14)
    a4 = oracle_mod.softmax(np.full((1, 1, 1, 16), 0.3), 4, 4)
    np.testing.assert_allclose(a4, 1.0 / 16, rtol=1e-15)
    big = oracle_mod.softmax(np.array([[[[1000.0, 0.0]]]]), 1, 2)
    assert np.isfinite(big).all() and abs(big.ravel()[0] - 1.0) < 1e-15


# -------------------------------------------------- library special case ---

def _grid_sample_reference(value, shapes, starts, loc, attn):
    """Per-level torch grid_sample (bilinear, zeros, align_corners=False) on
    grid = 2*loc - 1, weighted by A and summed -- the reduction
    cf-1.com/news/4799680 §5.3 describes, written against torch's documented
    API in float64 with autograd for the gradients."""
    B, S, M, D = value.shape
    _, Q, _, L, K, _ = loc.shape
    out = 0
    for l in range(L):
        H, W = int(shapes[l, 0]), int(shapes[l, 1])
        s0 = int(starts[l])
        v = value[:, s0:s0 + H * W].reshape(B, H, W, M, D).permute(0, 3, 4, 1, 2).reshape(B * M, D, H, W)
        grid = (2 * loc[:, :, :, l] - 1).permute(0, 2, 1, 3, 4).reshape(B * M, Q, K, 2)
        smp = torch.nn.functional.grid_sample(v, grid, mode="bilinear", padding_mode="zeros",
                                              align_corners=False)  # [B*M, D, Q, K]
        smp = smp.reshape(B, M, D, Q, K)
        a = attn[:, :, :, l].permute(0, 2, 1, 3).reshape(B, M, 1, Q, K)
        out = out + (smp * a).sum(-1)
    return out.permute(0, 3, 1, 2)  # [B, Q, M, D]


@pytest.mark.parametrize("name", ["tiny_f32", "ragged"])
def test_matches_torch_grid_sample(oracle_mod, name):
    if name == "tiny_f32":
        w = wl.WORKLOADS["tiny_f32"]
    else:
        w = wl.custom("ragged", 2, [(7, 13), (4, 6), (1, 3)], 23, 3, 5, 3, offset_sigma=2.5)
    x = wl.generate(w)
    v = torch.tensor(x.value_f64(), requires_grad=True)
    loc = torch.tensor(x.sampling_locations.astype(np.float64), requires_grad=True)
    a = torch.tensor(x.attention_weights.astype(np.float64), requires_grad=True)
    g = torch.tensor(x.grad_output_f64())
    out_t = _grid_sample_reference(v, x.spatial_shapes, x.level_start_index, loc, a)
    (out_t * g).sum().backward()
    out = oracle_mod.forward(x.value_f64(), x.spatial_shapes, x.level_start_index,
                             x.sampling_locations, x.attention_weights)
    np.testing.assert_allclose(out, out_t.detach().numpy(), rtol=1e-12, atol=1e-12)
    gv, gl, ga = oracle_mod.backward(x.value_f64(), x.spatial_shapes, x.level_start_index,
                                     x.sampling_locations, x.attention_weights, x.grad_output_f64())
    np.testing.assert_allclose(gv, v.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ga, a.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gl, loc.grad.numpy(), rtol=1e-10, atol=1e-10)


def test_encoder_sample_against_grid_sample(oracle_mod):
    """A slice of the Deformable-DETR encoder workload (first 300 queries of
    the 4-level 100x167 .. 13x21 map) against the grid_sample reduction."""
    w = wl.WORKLOADS["detr_encoder_f32"]
    x = wl.generate(w)
    q = slice(0, 300)
    loc = np.ascontiguousarray(x.sampling_locations[:, q].astype(np.float64))
    a = np.ascontiguousarray(x.attention_weights[:, q].astype(np.float64))
    out = oracle_mod.forward(x.value_f64(), x.spatial_shapes, x.level_start_index, loc, a)
    out_t = _grid_sample_reference(torch.tensor(x.value_f64()), x.spatial_shapes,
                                   x.level_start_index, torch.tensor(loc), torch.tensor(a))
    np.testing.assert_allclose(out, out_t.numpy(), rtol=1e-12, atol=1e-12)
