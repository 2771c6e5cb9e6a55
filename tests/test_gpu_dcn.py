"""DCNv3 core (msda_dcn_forward / msda_dcn_backward through the C ABI) against
the oracle's DCNv3 core on the same seeded inputs: the full-size layers, then
kernel sizes, strides, paddings, dilations, channel counts and dtypes that
reach every set-up path of the kernels (per-group for K = 9, 25, 49;
warp-wide for power-of-two K)."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, value_tensor

pytestmark = pytest.mark.gpu

TOL_S8 = {"row": 1e-2, "f32": 1e-5}


def _upload(x: wl.DcnInputs):
    w = x.workload
    return dict(input=value_tensor(x.input, w.dtype), offset=torch.from_numpy(x.offset).cuda(),
                mask=torch.from_numpy(x.mask).cuda(),
                grad_output=value_tensor(x.grad_output, w.dtype))


def _run(w: wl.DcnWorkload, x: wl.DcnInputs = None):
    x = x or wl.generate_dcn(w)
    t = _upload(x)
    geo = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dilation=w.dil)
    inp, scale = t["input"], None
    v64 = x.input_f64()
    if w.dtype == "s8":
        inp, scale = msda.quantize_value_s8(t["input"].flatten(1, 2))
        inp = inp.view(t["input"].shape)
        q, s = oracle.quantize_value_s8(x.input.reshape(w.N, w.H * w.W, w.G, w.C))
        assert np.array_equal(inp.cpu().numpy().reshape(q.shape), q)
        v64 = oracle.dequantize_value_s8(q, s).reshape(v64.shape)
    y = msda.dcn_forward(inp, t["offset"], t["mask"], value_scale=scale, **geo)
    gx, goff, gm = msda.dcn_backward(inp, t["offset"], t["mask"], t["grad_output"],
                                     value_scale=scale, **geo)
    assert msda.device_status() == 0
    og = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dil=w.dil)
    ry = oracle.dcn_forward(v64, x.offset, x.mask, **og)
    rgx, rgoff, rgm = oracle.dcn_backward(v64, x.offset, x.mask, x.grad_output_f64(), **og)
    if w.dtype == "s8":
        tol_row, tol = TOL_S8["row"], TOL_S8["f32"]
    else:
        tol_row = tol = TOL[w.dtype]
    return [assert_close(y, ry, tol_row, f"{w.name} output"),
            assert_close(gx, rgx, tol, f"{w.name} grad_input"),
            assert_close(goff, rgoff, tol, f"{w.name} grad_offset"),
            assert_close(gm, rgm, tol, f"{w.name} grad_mask")]


@pytest.mark.parametrize("name", sorted(wl.DCN_WORKLOADS))
def test_dcn_full_size(name):
    errs = _run(wl.DCN_WORKLOADS[name])
    print(f"{name}: errors {['%.2e' % e for e in errs]}")


EDGE = [
    # name, N, H, W, G, C, kernel, stride, pad, dil, dtype, sigma
    ("k3_s1_f32", 2, 13, 17, 3, 16, (3, 3), (1, 1), (1, 1), (1, 1), "f32", 1.0),
    ("k3_s2_f32", 2, 13, 17, 2, 32, (3, 3), (2, 2), (1, 1), (1, 1), "f32", 1.5),
    ("k5_dil2_bf16", 1, 21, 19, 2, 16, (5, 5), (1, 1), (4, 4), (2, 2), "bf16", 1.0),
    ("k7_f32", 1, 15, 12, 2, 8, (7, 7), (1, 1), (3, 3), (1, 1), "f32", 2.0),
    ("k1_nopad_f32", 2, 9, 11, 4, 64, (1, 1), (1, 1), (0, 0), (1, 1), "f32", 1.0),
    ("k2_warp_setup_f32", 1, 10, 10, 2, 16, (2, 2), (1, 1), (0, 0), (1, 1), "f32", 1.0),
    ("k4x8_warp_setup_bf16", 1, 12, 20, 2, 16, (4, 8), (1, 1), (2, 4), (1, 1), "bf16", 1.0),
    ("asym_stride_pad", 1, 16, 23, 2, 16, (3, 5), (2, 1), (0, 2), (1, 2), "f32", 1.0),
    ("far_offsets_f32", 1, 9, 9, 2, 16, (3, 3), (1, 1), (1, 1), (1, 1), "f32", 6.0),
    ("k3_s8", 2, 13, 17, 3, 16, (3, 3), (1, 1), (1, 1), (1, 1), "s8", 1.0),
    ("k7_s8_c128", 1, 11, 10, 2, 128, (7, 7), (1, 1), (3, 3), (1, 1), "s8", 1.0),
    ("c256_bf16", 1, 6, 7, 1, 256, (3, 3), (1, 1), (1, 1), (1, 1), "bf16", 1.0),
]


@pytest.mark.parametrize("spec", EDGE, ids=[e[0] for e in EDGE])
def test_dcn_edge_shapes(spec):
    name, N, H, W, G, C, k, s, p, d, dtype, sigma = spec
    _run(wl.custom_dcn(name, N, H, W, G, C, k, s, p, d, dtype, sigma, index=700 + EDGE.index(spec)))


def test_dcn_zero_offsets_match_torch_depthwise_conv():
    """With zero offsets and masks shared over positions the core is a
    depthwise convolution: compare the CUDA path with torch's conv2d."""
    N, H, W, G, C = 2, 14, 18, 4, 16
    g = torch.Generator().manual_seed(5)
    x = torch.randn(N, H, W, G, C, generator=g).cuda()
    taps = torch.randn(G, 9, generator=g)
    off = torch.zeros(N, H, W, G, 9, 2, device="cuda")
    mask = taps.cuda()[None, None, None].expand(N, H, W, G, 9).contiguous()
    y = msda.dcn_forward(x, off, mask, kernel=3, stride=1, pad=1, dilation=1)
    xt = x.permute(0, 3, 4, 1, 2).reshape(N, G * C, H, W).double().cpu()
    wt = taps.reshape(G, 1, 3, 3).repeat_interleave(C, 0).double()
    ref = torch.nn.functional.conv2d(xt, wt, padding=1, groups=G * C)
    ref = ref.reshape(N, G, C, H, W).permute(0, 3, 4, 1, 2)
    assert_close(y, ref.numpy(), 1e-5, "zero-offset DCN vs depthwise conv2d")


def test_dcn_host_checks():
    x = torch.zeros(1, 5, 5, 2, 16, device="cuda")
    off = torch.zeros(1, 5, 5, 2, 9, 2, device="cuda")
    m = torch.zeros(1, 5, 5, 2, 9, device="cuda")
    with pytest.raises(msda.MsdaError):  # 3 x 33 kernel: kernel_w > 32
        msda.dcn_forward(x, torch.zeros(1, 5, 5, 2, 99, 2, device="cuda"),
                         torch.zeros(1, 5, 5, 2, 99, device="cuda"), kernel=(3, 33), pad=(1, 16))
    with pytest.raises(ValueError):  # offsets of the wrong shape
        msda.dcn_forward(x, off[:, :4], m, kernel=3, pad=1)
    y = msda.dcn_forward(x, off, m, kernel=3, pad=1)
    assert y.shape == (1, 5, 5, 2, 16) and not y.any()


def test_dcn_autograd_wrapper():
    w = wl.custom_dcn("dcn_autograd", 2, 9, 11, 2, 16, (3, 3), (1, 1), (1, 1), (1, 1), "f32", 1.0,
                      index=790)
    x = wl.generate_dcn(w)
    t = _upload(x)
    inp = t["input"].clone().requires_grad_(True)
    off = t["offset"].clone().requires_grad_(True)
    m = t["mask"].clone().requires_grad_(True)
    y = msda.dcnv3_core(inp, off, m, kernel=3, stride=1, pad=1, dilation=1)
    Ho, Wo = w.out_hw
    assert y.shape == (2, Ho, Wo, 32)
    (y * t["grad_output"].flatten(3)).sum().backward()
    og = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dil=w.dil)
    rgx, rgoff, rgm = oracle.dcn_backward(x.input_f64(), x.offset, x.mask, x.grad_output_f64(), **og)
    assert_close(inp.grad, rgx, 1e-5, "autograd grad_input")
    assert_close(off.grad, rgoff, 1e-5, "autograd grad_offset")
    assert_close(m.grad, rgm, 1e-5, "autograd grad_mask")
