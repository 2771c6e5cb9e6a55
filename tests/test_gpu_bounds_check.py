"""The checked build (MSDA_BOUNDS_CHECK=1: every corner row a kernel reads or
reduces into is tested against its tensor, a violation recorded as
MSDA_ERR_DEVICE_BOUNDS and the access skipped) runs every kernel family on
full-size and edge workloads: the status stays clean and the results match
the oracle.  This stands in for a memory checker, which is closed here."""
import ctypes

import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import _lib, build
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, oracle_fused, oracle_nonfused, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked_lib():
    path = build.build_checked()
    saved = _lib._lib
    _lib._lib = None
    lib = _lib.load(path)
    yield lib
    _lib._lib = saved


def _attention(w):
    x = wl.generate(w)
    t = upload(x)
    geo = (t["spatial_shapes"], t["level_start_index"])
    out = msda.forward(t["value"], *geo, t["sampling_locations"], t["attention_weights"])
    gv, gl, ga = msda.backward(t["value"], *geo, t["sampling_locations"], t["attention_weights"],
                               t["grad_output"])
    fout = msda.fused_forward(t["value"], *geo, t["reference_points"], t["sampling_offsets"],
                              t["attention_logits"])
    fgv, fgref, fgoff, fglog = msda.fused_backward(t["value"], *geo, t["reference_points"],
                                                   t["sampling_offsets"], t["attention_logits"],
                                                   t["grad_output"])
    assert msda.device_status() == 0
    tol = TOL[w.dtype]
    r = oracle_nonfused(x)
    for g, ref, what in zip((out, gv, gl, ga), r, ("out", "grad_value", "grad_loc", "grad_attn")):
        assert_close(g, ref, tol, f"checked {w.name} {what}")
    rf = oracle_fused(x)
    for g, ref, what in zip((fout, fgv, fgref, fgoff, fglog), (rf[0],) + rf[2:],
                            ("out", "grad_value", "grad_ref", "grad_off", "grad_logits")):
        assert_close(g, ref, tol, f"checked fused {w.name} {what}")


@pytest.mark.parametrize("name", ["detr_encoder_f32", "stress_1080p_k8_bf16"])
def test_checked_build_full_size(checked_lib, name):
    assert _lib.load() is checked_lib
    _attention(wl.WORKLOADS[name])


@pytest.mark.parametrize("spec", [
    ("chk_d8", 2, [(7, 9), (3, 5)], 37, 3, 8, 3, "f32", "uniform", 2.0),
    ("chk_one_pixel", 1, [(1, 1), (1, 3), (2, 1)], 40, 8, 32, 4, "bf16", "uniform", 0.7),
    ("chk_far", 1, [(10, 12), (5, 6)], 64, 4, 64, 4, "f32", "uniform", 40.0),
    ("chk_k32", 1, [(20, 30), (10, 15), (5, 8), (3, 4)], 45, 2, 256, 32, "bf16", "uniform", 3.0),
], ids=lambda s: s[0])
def test_checked_build_edges(checked_lib, spec):
    name, B, levels, Q, M, D, K, dtype, ref, sigma = spec
    _attention(wl.custom(name, B, levels, Q, M, D, K, dtype, ref, sigma, 1.0, index=900))


def test_checked_build_int8_and_dcn(checked_lib):
    w = wl.DCN_WORKLOADS["dcnv3_k7_bf16"]
    x = wl.generate_dcn(w)
    inp = torch.from_numpy(x.input.view("int16")).cuda().view(torch.bfloat16)
    q, s = msda.quantize_value_s8(inp.flatten(1, 2))
    q = q.view(inp.shape)
    off, m = torch.from_numpy(x.offset).cuda(), torch.from_numpy(x.mask).cuda()
    gy = torch.from_numpy(x.grad_output.view("int16")).cuda().view(torch.bfloat16)
    geo = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dilation=w.dil)
    y = msda.dcn_forward(q, off, m, value_scale=s, **geo)
    gx, goff, gm = msda.dcn_backward(q, off, m, gy, value_scale=s, **geo)
    assert msda.device_status() == 0
    rq, rs = oracle.quantize_value_s8(x.input.reshape(w.N, w.H * w.W, w.G, w.C))
    v64 = oracle.dequantize_value_s8(rq, rs).reshape(x.input.shape)
    og = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dil=w.dil)
    assert_close(y, oracle.dcn_forward(v64, x.offset, x.mask, **og), 1e-2, "checked int8 dcn out")
    rgx, rgoff, rgm = oracle.dcn_backward(v64, x.offset, x.mask, x.grad_output_f64(), **og)
    assert_close(gx, rgx, 1e-5, "checked int8 dcn grad_input")
    assert_close(goff, rgoff, 1e-5, "checked int8 dcn grad_offset")
    assert_close(gm, rgm, 1e-5, "checked int8 dcn grad_mask")


def test_checked_build_fp8_decoder(checked_lib):
    """FP8 value on the decoder's shape (rows split over lane groups in the
    forward) through the four operator calls."""
    w = wl.custom("chk_fp8_decoder", 2, [(100, 167), (50, 84), (25, 42), (13, 21)], 300, 8, 32, 4,
                  "e4m3", "uniform_inner", 4.0, 1.0, index=901)
    x = wl.generate(w)
    t = upload(x)
    q, s = msda.quantize_value_e4m3(t["value"])
    geo = (t["spatial_shapes"], t["level_start_index"])
    out = msda.forward(q, *geo, t["sampling_locations"], t["attention_weights"], value_scale=s)
    gv, gl, ga = msda.backward(q, *geo, t["sampling_locations"], t["attention_weights"],
                               t["grad_output"], value_scale=s)
    fout = msda.fused_forward(q, *geo, t["reference_points"], t["sampling_offsets"],
                              t["attention_logits"], value_scale=s)
    fgv, fgref, fgoff, fglog = msda.fused_backward(q, *geo, t["reference_points"], t["sampling_offsets"],
                                                   t["attention_logits"], t["grad_output"], value_scale=s)
    assert msda.device_status() == 0
    rq, rs = oracle.quantize_value_e4m3(x.value)
    x.value = oracle.dequantize_value_e4m3(rq, rs)  # the oracle samples decode(code) * scale
    r = oracle_nonfused(x)
    for g, ref, what, tol in zip((out, gv, gl, ga), r, ("out", "grad_value", "grad_loc", "grad_attn"),
                                 (1e-2, 1e-5, 1e-5, 1e-5)):
        assert_close(g, ref, tol, f"checked fp8 decoder {what}")
    rf = oracle_fused(x)
    for g, ref, what, tol in zip((fout, fgv, fgref, fgoff, fglog), (rf[0],) + rf[2:],
                                 ("out", "grad_value", "grad_ref", "grad_off", "grad_logits"),
                                 (1e-2, 1e-5, 1e-5, 1e-5, 1e-5)):
        assert_close(g, ref, tol, f"checked fp8 decoder fused {what}")
