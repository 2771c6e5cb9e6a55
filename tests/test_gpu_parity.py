"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded
inputs, element by element.  Needs a B200 (sm_100a)."""
import numpy as np
import pytest
import torch

import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, bf16_round, oracle_fused, oracle_nonfused, upload

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    torch.cuda.init()

_cache = {}


def _inputs(w: wl.Workload):
    if w.name not in _cache:
        _cache.clear()
        _cache[w.name] = {"x": wl.generate(w)}
    return _cache[w.name]["x"]


def _oracle(w: wl.Workload, x, which):
    """Oracle results of the cached workload inputs (computed once per
    workload), or of ad-hoc inputs x."""
    fn = oracle_nonfused if which == "nonfused" else oracle_fused
    if w.name in _cache and _cache[w.name]["x"] is x:
        c = _cache[w.name]
        if which not in c:
            c[which] = fn(x)
        return c[which]
    return fn(x)


def _run_nonfused(w: wl.Workload, x=None, merge=False):
    x = x or _inputs(w)
    t = upload(x)
    out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                       t["sampling_locations"], t["attention_weights"])
    gv, gl, ga = msda.backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                               t["sampling_locations"], t["attention_weights"], t["grad_output"],
                               merge_reductions=merge)
    assert msda.device_status() == 0
    ref = _oracle(w, x, "nonfused")
    tol = TOL[w.dtype]
    errs = [assert_close(out, ref[0], tol, f"{w.name} out"),
            assert_close(gv, ref[1], tol, f"{w.name} grad_value"),
            assert_close(gl, ref[2], tol, f"{w.name} grad_sampling_locations"),
            assert_close(ga, ref[3], tol, f"{w.name} grad_attention_weights")]
    return errs


def _run_fused(w: wl.Workload, x=None, want_ref=True, merge=False):
    x = x or _inputs(w)
    t = upload(x)
    out, attn = msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                                   t["reference_points"], t["sampling_offsets"],
                                   t["attention_logits"], return_attention_weights=True)
    gv, gref, goff, glog = msda.fused_backward(t["value"], t["spatial_shapes"],
                                               t["level_start_index"], t["reference_points"],
                                               t["sampling_offsets"], t["attention_logits"],
                                               t["grad_output"],
                                               want_grad_reference_points=want_ref,
                                               merge_reductions=merge)
    assert msda.device_status() == 0
    r_out, r_a, r_gv, r_gref, r_goff, r_glog = _oracle(w, x, "fused")
    tol = TOL[w.dtype]
    errs = [assert_close(out, r_out, tol, f"{w.name} fused out"),
            assert_close(attn, r_a, tol, f"{w.name} fused attention weights"),
            assert_close(gv, r_gv, tol, f"{w.name} fused grad_value"),
            assert_close(goff, r_goff, tol, f"{w.name} fused grad_sampling_offsets"),
            assert_close(glog, r_glog, tol, f"{w.name} fused grad_attention_logits")]
    if want_ref:
        errs.append(assert_close(gref, r_gref, tol, f"{w.name} fused grad_reference_points"))
    else:
        assert gref is None
    return errs


ALL = sorted((n for n in wl.WORKLOADS if wl.WORKLOADS[n].dtype not in ("s8", "e4m3")),
             key=lambda n: wl.WORKLOADS[n].index)  # INT8 value: tests/test_gpu_int8.py


@pytest.mark.parametrize("merge", [False, True], ids=["direct", "merged"])
@pytest.mark.parametrize("name", ALL)
def test_full_size(name, merge):
    """Every output of msda_forward / msda_backward and of msda_fused_forward /
    msda_fused_backward at the workload's full size, with the launch
    configuration the bench times (the library picks it from the sizes);
    the backward with direct (default) and with merged grad_value
    reductions."""
    w = wl.WORKLOADS[name]
    e1 = _run_nonfused(w, merge=merge)
    e2 = _run_fused(w, merge=merge)
    print(f"{name}: non-fused errors {['%.2e' % e for e in e1]} fused errors {['%.2e' % e for e in e2]}")


# -------------------------------------------------------------- edge shapes --

EDGE = [
    # (name, B, levels, Q, M, D, K, dtype, ref, sigma)
    ("d8_f32", 2, [(7, 9), (3, 5)], 37, 3, 8, 3, "f32", "uniform", 2.0),
    ("d8_bf16", 2, [(7, 9), (3, 5)], 37, 3, 8, 3, "bf16", "uniform", 2.0),
    ("d16_f32", 1, [(11, 6), (5, 3), (2, 2)], 50, 2, 16, 4, "f32", "uniform", 1.5),
    ("d16_bf16", 1, [(11, 6), (5, 3), (2, 2)], 50, 2, 16, 4, "bf16", "uniform", 1.5),
    ("d64_f32", 2, [(13, 17), (7, 9)], 29, 4, 64, 2, "f32", "uniform", 3.0),
    ("d64_bf16", 2, [(13, 17), (7, 9)], 29, 4, 64, 2, "bf16", "uniform", 3.0),
    ("d128_f32", 1, [(9, 10)], 33, 2, 128, 5, "f32", "uniform", 2.0),
    ("d128_bf16", 1, [(9, 10)], 33, 2, 128, 5, "bf16", "uniform", 2.0),
    ("d256_f32", 1, [(6, 7), (3, 4)], 21, 2, 256, 3, "f32", "uniform", 2.0),
    ("d256_bf16", 1, [(6, 7), (3, 4)], 21, 2, 256, 3, "bf16", "uniform", 2.0),
    ("single_level_single_point", 3, [(15, 23)], 101, 5, 32, 1, "f32", "uniform", 1.0),
    ("one_pixel_levels", 1, [(1, 1), (1, 3), (2, 1)], 40, 8, 32, 4, "f32", "uniform", 0.7),
    ("k32_l4_many_points", 1, [(20, 30), (10, 15), (5, 8), (3, 4)], 45, 2, 32, 32, "f32", "uniform", 3.0),
    ("l16_k8", 1, [(4 + l, 3 + (l % 5)) for l in range(16)], 19, 2, 32, 8, "bf16", "uniform", 2.0),
    ("ragged_tail_encoder", 2, [(11, 13), (6, 7), (3, 4)], None, 8, 32, 4, "f32", "pixel_centre", 2.0),
    ("ragged_tail_bf16", 3, [(11, 13), (6, 7), (3, 4)], None, 8, 32, 4, "bf16", "pixel_centre", 2.0),
    ("mostly_out_of_range", 1, [(10, 12), (5, 6)], 64, 4, 32, 4, "f32", "uniform", 40.0),
]


def _edge(spec):
    name, B, levels, Q, M, D, K, dtype, ref, sigma = spec
    return wl.custom(name, B, levels, Q, M, D, K, dtype, ref, sigma, 1.0, index=200 + EDGE.index(spec))


@pytest.mark.parametrize("merge", [False, True], ids=["direct", "merged"])
@pytest.mark.parametrize("spec", EDGE, ids=[e[0] for e in EDGE])
def test_edge_shapes(spec, merge):
    w = _edge(spec)
    x = wl.generate(w)
    _run_nonfused(w, x, merge=merge)
    _run_fused(w, x, want_ref=(spec[0] != "d8_f32"), merge=merge)


def test_integer_pixel_coordinates():
    """Zero offsets at pixel centres of power-of-two levels put every sample on
    an exact integer coordinate (fx = fy = 0): the one-sided derivative of the
    cell floor(x) is used on both sides, and the forward returns the pixel."""
    w = wl.custom("integer_px", 1, [(8, 16), (4, 8), (2, 4)], None, 2, 32, 1, "f32",
                  "pixel_centre", 0.0, 1.0, index=300)
    x = wl.generate(w)
    x.sampling_offsets[:] = 0.0
    _run_fused(w, x)


def test_exact_borders_are_outside():
    """x = -1 or x = W (and likewise for y) is outside: zero output and zero
    gradients for that sample."""
    w = wl.custom("borders", 1, [(4, 8)], 4, 1, 8, 2, "f32", "uniform", 1.0, index=301)
    x = wl.generate(w)
    W, H = 8.0, 4.0
    pts = [(-0.5 / W, 0.5), (1.0 + 0.5 / W, 0.5), (0.5, -0.5 / H), (0.5, 1.0 + 0.5 / H)]
    for q, p in enumerate(pts):
        x.sampling_locations[0, q, 0, 0, 0] = p
    t = upload(x)
    out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                       t["sampling_locations"], t["attention_weights"])
    ref = oracle_nonfused(x)
    assert_close(out, ref[0], 1e-6, "borders out")
    gv, gl, ga = msda.backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                               t["sampling_locations"], t["attention_weights"], t["grad_output"])
    assert gl[0, :, 0, 0, 0].abs().max().item() == 0.0
    assert ga[0, :, 0, 0, 0].abs().max().item() == 0.0
    assert_close(gl, ref[2], 1e-5, "borders grad_loc")


def test_empty_batch_and_queries():
    for B, Q in [(0, 5), (2, 0)]:
        w = wl.custom("empty", max(B, 1), [(4, 5), (2, 3)], max(Q, 1), 2, 16, 2, "f32", index=302)
        x = wl.generate(w)
        t = upload(x)
        v = t["value"][:B] if B == 0 else t["value"]
        S = v.shape[1]
        loc = torch.zeros((B, Q, 2, 2, 2, 2), device="cuda")
        a = torch.zeros((B, Q, 2, 2, 2), device="cuda")
        out = msda.forward(v, t["spatial_shapes"], t["level_start_index"], loc, a)
        assert out.shape == (B, Q, 2, 16)
        g = torch.zeros((B, Q, 2, 16), device="cuda")
        gv, gl, ga = msda.backward(v, t["spatial_shapes"], t["level_start_index"], loc, a, g)
        assert gv.shape == (B, S, 2, 16)
        if gv.numel():
            assert gv.abs().max().item() == 0.0
    assert msda.device_status() == 0


def test_forward_is_deterministic():
    w = wl.WORKLOADS["detr_encoder_f32"]
    t = upload(_inputs(w))
    o1 = msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                            t["reference_points"], t["sampling_offsets"], t["attention_logits"])
    o2 = msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                            t["reference_points"], t["sampling_offsets"], t["attention_logits"])
    assert torch.equal(o1, o2)


def test_adjoint_identity_full_size():
    """<grad_value, value> = <g, out> at full size: grad_value is the adjoint of
    the forward in value (holds at any size)."""
    w = wl.WORKLOADS["stress_1080p_k8_bf16"]
    t = upload(_inputs(w))
    out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                       t["sampling_locations"], t["attention_weights"])
    gv, _, ga = msda.backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                              t["sampling_locations"], t["attention_weights"], t["grad_output"])
    v = t["value"].double()
    g = t["grad_output"].double()
    lhs = (gv.double() * v).sum().item()
    lhs_a = (ga.double() * t["attention_weights"].double()).sum().item()
    # out is rounded to bf16 here; compare against the float32 path instead
    rhs = (g * out.double()).sum().item()
    scale = (g.abs() * out.double().abs()).sum().item()
    assert abs(lhs - rhs) <= 1e-2 * scale
    assert abs(lhs_a - lhs) <= 1e-4 * scale


def test_grad_value_bf16_output():
    """MSDA_GRAD_VALUE_BF16: grad_value written as bf16 is the oracle's
    float64 grad_value rounded to bf16, up to one rounding step (the float32
    sum and the float64 one can round to neighbouring bf16 values), and one
    bf16 step is at most 2^-7 of the value: the elementwise error against
    the rounded oracle stays within 2^-7."""
    w = wl.WORKLOADS["detr_decoder_bf16"]
    x = _inputs(w)
    t = upload(x)
    args = (t["value"], t["spatial_shapes"], t["level_start_index"], t["sampling_locations"],
            t["attention_weights"], t["grad_output"])
    gv32, gl32, ga32 = msda.backward(*args)
    gv16, gl16, ga16 = msda.backward(*args, grad_value_dtype=torch.bfloat16)
    assert gv16.dtype == torch.bfloat16
    ref = _oracle(w, x, "nonfused")
    assert_close(gv16, bf16_round(ref[1]), 2.0 ** -7, "bf16 grad_value vs rounded oracle",
                 elem_tol=2.0 ** -7)
    assert_close(gv16, ref[1], TOL["bf16"], "bf16 grad_value vs oracle")
    assert torch.equal(gl16, gl32) and torch.equal(ga16, ga32)
    gvf, _, _, _ = msda.fused_backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                                       t["reference_points"], t["sampling_offsets"],
                                       t["attention_logits"], t["grad_output"],
                                       grad_value_dtype=torch.bfloat16)
    assert gvf.dtype == torch.bfloat16
    rf = _oracle(w, x, "fused")
    assert_close(gvf, bf16_round(rf[2]), 2.0 ** -7, "fused bf16 grad_value vs rounded oracle",
                 elem_tol=2.0 ** -7)


def test_inconsistent_geometry_sets_device_status():
    """A level_start_index that does not match spatial_shapes is caught by the
    kernels (no fault): the work is skipped and the status word says so."""
    w = wl.WORKLOADS["tiny_f32"]
    t = upload(_inputs(w))
    assert msda.device_status() == 0
    bad_start = t["level_start_index"].clone()
    bad_start[1] += 1
    msda.forward(t["value"], t["spatial_shapes"], bad_start, t["sampling_locations"],
                 t["attention_weights"])
    assert msda.device_status() == 4
    assert msda.device_status() == 0  # cleared by the read
    bad_shapes = t["spatial_shapes"].clone()
    bad_shapes[0, 0] = 0
    msda.fused_backward(t["value"], bad_shapes, t["level_start_index"], t["reference_points"],
                        t["sampling_offsets"], t["attention_logits"], t["grad_output"])
    assert msda.device_status() == 4


def test_host_validation_errors():
    w = wl.WORKLOADS["tiny_f32"]
    t = upload(_inputs(w))
    with pytest.raises(msda.MsdaError) as e:
        # head_dim 24 is not a supported size
        v = torch.zeros((1, 80, 2, 24), device="cuda")
        msda.forward(v, t["spatial_shapes"], t["level_start_index"], t["sampling_locations"],
                     t["attention_weights"])
    assert e.value.status == 2
    with pytest.raises(ValueError):
        msda.forward(t["value"][:, :, :, :4], t["spatial_shapes"], t["level_start_index"],
                     t["sampling_locations"], t["attention_weights"])
    with pytest.raises(ValueError):
        msda.forward(t["value"].cpu(), t["spatial_shapes"], t["level_start_index"],
                     t["sampling_locations"], t["attention_weights"])


def test_autograd_wrappers():
    w = wl.custom("autograd", 2, [(6, 9), (3, 5)], 11, 2, 16, 3, "f32", index=303)
    x = wl.generate(w)
    t = upload(x)
    v = t["value"].clone().requires_grad_(True)
    loc = t["sampling_locations"].clone().requires_grad_(True)
    a = t["attention_weights"].clone().requires_grad_(True)
    out = msda.ms_deform_attn(v, t["spatial_shapes"], t["level_start_index"], loc, a)
    assert out.shape == (2, 11, 32)
    (out * t["grad_output"].flatten(2)).sum().backward()
    ref = oracle_nonfused(x)
    assert_close(v.grad, ref[1], 1e-5, "autograd grad_value")
    assert_close(loc.grad, ref[2], 1e-5, "autograd grad_loc")
    # the usual call site with a trailing im2col_step (accepted, ignored)
    out64 = msda.MSDeformAttnFunction.apply(t["value"], t["spatial_shapes"], t["level_start_index"],
                                            t["sampling_locations"], t["attention_weights"], 64)
    assert torch.equal(out64.flatten(2), out.detach())
    assert_close(a.grad, ref[3], 1e-5, "autograd grad_attn")
    ref_pts = t["reference_points"].clone().requires_grad_(True)
    off = t["sampling_offsets"].clone().requires_grad_(True)
    logit = t["attention_logits"].clone().requires_grad_(True)
    v.grad = None
    out = msda.MSDeformAttnFusedFunction.apply(v, t["spatial_shapes"], t["level_start_index"],
                                               ref_pts, off, logit)
    (out * t["grad_output"]).sum().backward()
    rf = oracle_fused(x)
    assert_close(v.grad, rf[2], 1e-5, "autograd fused grad_value")
    assert_close(ref_pts.grad, rf[3], 1e-5, "autograd fused grad_ref")
    assert_close(off.grad, rf[4], 1e-5, "autograd fused grad_off")
    assert_close(logit.grad, rf[5], 1e-5, "autograd fused grad_logits")


def test_nondefault_stream():
    w = wl.WORKLOADS["tiny_f32"]
    x = _inputs(w)
    t = upload(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                           t["sampling_locations"], t["attention_weights"])
    s.synchronize()
    assert_close(out, oracle_nonfused(x)[0], 1e-5, "stream out")


def test_bounded_wait_reports_timeout_and_context_survives():
    """With MSDA_STAGE_INPUTS the forward stages its inputs with bulk copies
    and waits for them with a bounded poll.  With MSDA_TEST_WITHHOLD_COPY the
    copy is armed but never issued: the wait runs out, the kernel reports
    MSDA_ERR_DEVICE_TIMEOUT and returns, and the next call works."""
    import ctypes
    from scale_deformable_attention_msdeformattn_b200 import _lib
    w = wl.custom("timeout", 1, [(16, 16), (8, 8)], 64, 2, 32, 2, "f32", index=304)
    x = wl.generate(w)
    t = upload(x)
    out = torch.empty((1, 64, 2, 32), device="cuda")
    prob = _lib.Problem(1, w.S, 64, 2, 32, 2, 2, _lib.MSDA_F32,
                        _lib.MSDA_STAGE_INPUTS | _lib.MSDA_TEST_WITHHOLD_COPY)
    p = lambda z: ctypes.c_void_p(z.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert msda.device_status() == 0
    st = _lib.load().msda_forward(ctypes.byref(prob), p(t["value"]), p(t["spatial_shapes"]),
                                  p(t["level_start_index"]), p(t["sampling_locations"]),
                                  p(t["attention_weights"]), p(out), stream)
    assert st == 0
    assert msda.device_status() == _lib.MSDA_ERR_DEVICE_TIMEOUT
    # the context is intact: a normal call succeeds and is correct, staged too
    out2 = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                        t["sampling_locations"], t["attention_weights"])
    assert msda.device_status() == 0
    assert_close(out2, oracle_nonfused(x)[0], 1e-5, "after timeout")
    prob.flags = _lib.MSDA_STAGE_INPUTS
    out3 = torch.empty_like(out)
    st = _lib.load().msda_forward(ctypes.byref(prob), p(t["value"]), p(t["spatial_shapes"]),
                                  p(t["level_start_index"]), p(t["sampling_locations"]),
                                  p(t["attention_weights"]), p(out3), stream)
    assert st == 0 and msda.device_status() == 0
    assert_close(out3, oracle_nonfused(x)[0], 1e-5, "staged forward")
