"""The MSDeformAttn layer (torch linear projections around the fused
kernels) against the same layer composed in float64 on the CPU with the
oracle as its core: output, input gradients and parameter gradients."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu


class _OracleCore(torch.autograd.Function):
    """The fused core in float64 on the CPU (the oracle), for autograd."""

    @staticmethod
    def forward(ctx, value, shapes, starts, ref, off, logits):
        ctx.save_for_backward(value, ref, off, logits)
        ctx.geo = (shapes.numpy(), starts.numpy())
        out, _, _ = oracle.fused_forward(value.numpy(), *ctx.geo, ref.numpy(), off.numpy(), logits.numpy())
        return torch.from_numpy(out)

    @staticmethod
    def backward(ctx, g):
        value, ref, off, logits = ctx.saved_tensors
        gv, gref, goff, glog = oracle.fused_backward(value.numpy(), *ctx.geo, ref.numpy(), off.numpy(),
                                                     logits.numpy(), g.contiguous().numpy())
        return (torch.from_numpy(gv), None, None, torch.from_numpy(gref), torch.from_numpy(goff),
                torch.from_numpy(glog))


def _reference(mod64, query, ref, x, shapes, starts, mask):
    B, Q, C = query.shape
    S = x.shape[1]
    M, L, K = mod64.n_heads, mod64.n_levels, mod64.n_points
    value = mod64.value_proj(x).masked_fill(mask[..., None], 0.0).reshape(B, S, M, C // M)
    off = mod64.sampling_offsets(query).reshape(B, Q, M, L, K, 2)
    logits = mod64.attention_weights(query).reshape(B, Q, M, L * K)
    out = _OracleCore.apply(value, shapes, starts, ref, off, logits)
    return mod64.output_proj(out.reshape(B, Q, C))


def test_layer_matches_float64_composition():
    torch.manual_seed(0)
    levels = [(16, 20), (8, 10), (4, 5), (2, 3)]
    shapes = torch.tensor(levels, dtype=torch.int64)
    starts = torch.from_numpy(wl.level_start_index(levels))
    B, Q, C, S = 2, 57, 64, int(sum(h * w for h, w in levels))
    mod = msda.MSDeformAttn(d_model=C, n_levels=4, n_heads=4, n_points=4)
    with torch.no_grad():  # offsets away from zero so that sampling moves
        mod.sampling_offsets.weight.normal_(0.0, 0.05)
        mod.sampling_offsets.bias.normal_(0.0, 1.0)
    mod64 = msda.MSDeformAttn(d_model=C, n_levels=4, n_heads=4, n_points=4).double()
    mod64.load_state_dict({k: v.double() for k, v in mod.state_dict().items()})
    query = torch.randn(B, Q, C, dtype=torch.float64)
    ref = torch.rand(B, Q, 2, dtype=torch.float64)
    x = torch.randn(B, S, C, dtype=torch.float64)
    mask = torch.zeros(B, S, dtype=torch.bool)
    mask[1, -7:] = True
    g = torch.randn(B, Q, C, dtype=torch.float64)

    mod = mod.cuda()
    qd = query.float().cuda().requires_grad_(True)
    rd = ref.float().cuda().requires_grad_(True)
    xd = x.float().cuda().requires_grad_(True)
    out = mod(qd, rd, xd, shapes.cuda(), starts.cuda(), mask.cuda())
    (out * g.float().cuda()).sum().backward()
    assert msda.device_status() == 0

    # the float32 inputs the GPU sees, widened
    q64 = query.float().double().requires_grad_(True)
    r64 = ref.float().double().requires_grad_(True)
    x64 = x.float().double().requires_grad_(True)
    ref_out = _reference(mod64, q64, r64, x64, shapes, starts, mask)
    (ref_out * g.float().double()).sum().backward()

    tol = 1e-4
    assert_close(out, ref_out.detach().numpy(), tol, "layer output")
    assert_close(qd.grad, q64.grad.numpy(), tol, "grad query")
    assert_close(rd.grad, r64.grad.numpy(), tol, "grad reference_points")
    assert_close(xd.grad, x64.grad.numpy(), tol, "grad input_flatten")
    for name in ("sampling_offsets", "attention_weights", "value_proj", "output_proj"):
        got = getattr(mod, name).weight.grad
        want = getattr(mod64, name).weight.grad.numpy()
        assert_close(got, want, tol, f"grad {name}.weight")
    # padded keys carry no value: their input rows get no gradient
    assert not xd.grad[1, -7:].any()
