"""Randomised shapes against the oracle: 48 seeded configurations drawn over
the supported ranges (B, level count and sizes, Q, M, D, K, dtype, reference
recipe, offset spread), each run through the non-fused and fused calls, every
fourth with a random query order and every fifth with INT8 value.  The draws
come from a fixed seed, so a failure names a reproducible configuration."""
import random

import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, oracle_fused, oracle_nonfused, upload

pytestmark = pytest.mark.gpu


def _configs(n=48, seed=20261202):
    r = random.Random(seed)
    out = []
    for i in range(n):
        L = r.randint(1, 5)
        K = r.choice([1, 2, 3, 4, 5, 8])
        if L * K > 128:
            K = 128 // L
        levels = [(r.randint(1, 23), r.randint(1, 23)) for _ in range(L)]
        D = r.choice([8, 16, 32, 64, 128, 256])
        M = r.randint(1, 9)
        B = r.randint(1, 3)
        ref = r.choice(["uniform", "uniform", "pixel_centre"])
        Q = None if ref == "pixel_centre" else r.randint(1, 90)
        if ref == "pixel_centre":  # Q = S: keep the oracle's work to seconds
            levels = [(min(h, 12), min(wd, 12)) for h, wd in levels]
            D = min(D, 64)
        dtype = r.choice(["f32", "bf16"])
        if i % 5 == 4:
            dtype = "s8"
        sigma = r.choice([0.5, 1.0, 2.0, 6.0, 30.0])
        out.append((f"fz{i}", B, levels, Q, M, D, K, dtype, ref, sigma, i % 4 == 3))
    return out


CONFIGS = _configs()


@pytest.mark.parametrize("spec", CONFIGS, ids=[c[0] for c in CONFIGS])
def test_random_shape(spec):
    name, B, levels, Q, M, D, K, dtype, ref, sigma, ordered = spec
    w = wl.custom(name, B, levels, Q, M, D, K, dtype, ref, sigma, 1.0, index=1000 + int(name[2:]))
    x = wl.generate(w)
    t = upload(x)
    geo = (t["spatial_shapes"], t["level_start_index"])
    order = None
    if ordered:
        g = torch.Generator().manual_seed(int(name[2:]))
        order = torch.randperm(w.B * w.num_queries, generator=g).to(torch.int32).cuda()
    value, scale = t["value"], None
    tol_row = tol = TOL["bf16" if dtype == "s8" else dtype]
    if dtype == "s8":
        value, scale = msda.quantize_value_s8(t["value"])
        q, s = oracle.quantize_value_s8(x.value)
        assert np.array_equal(value.cpu().numpy(), q) and np.array_equal(scale.cpu().numpy(), s)
        tol_row, tol = 1e-2, 1e-5
        x.value = oracle.dequantize_value_s8(q, s)  # the oracle samples q * scale (exact)
    out = msda.forward(value, *geo, t["sampling_locations"], t["attention_weights"],
                       query_order=order, value_scale=scale)
    gv, gl, ga = msda.backward(value, *geo, t["sampling_locations"], t["attention_weights"],
                               t["grad_output"], query_order=order, value_scale=scale)
    fout = msda.fused_forward(value, *geo, t["reference_points"], t["sampling_offsets"],
                              t["attention_logits"], query_order=order, value_scale=scale)
    fgv, fgref, fgoff, fglog = msda.fused_backward(value, *geo, t["reference_points"],
                                                   t["sampling_offsets"], t["attention_logits"],
                                                   t["grad_output"], query_order=order,
                                                   value_scale=scale)
    assert msda.device_status() == 0
    r = oracle_nonfused(x)
    for got, want, what, tl in zip((out, gv, gl, ga), r, ("out", "grad_value", "grad_loc", "grad_attn"),
                                   (tol_row, tol, tol, tol)):
        assert_close(got, want, tl, f"{name} {what}")
    rf = oracle_fused(x)
    for got, want, what, tl in zip((fout, fgv, fgref, fgoff, fglog), (rf[0],) + rf[2:],
                                   ("out", "grad_value", "grad_ref", "grad_off", "grad_logits"),
                                   (tol_row, tol, tol, tol, tol)):
        assert_close(got, want, tl, f"{name} fused {what}")
