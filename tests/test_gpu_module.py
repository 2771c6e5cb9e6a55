"""The MSDeformAttn layer on the GPU (tensor-core projections and fused query
head around the core) against the same layer composed in float64 on the CPU
from the oracle: output, input gradients and parameter gradients.

The layer computes in mixed precision: its projections take bf16 operands
(the float32 parameters and activations rounded to bf16, and in the backward
the gradient rows rounded to bf16) and accumulate in float32; it stores the
value tensor, the core's output rows and their gradient rows in bf16, and
its weight gradients come back from the bf16 GEMMs rounded to bf16.  The
float64 composition takes the same bf16-rounded operands and rounds at the
same points, so that the two differ only by accumulation order (and by the
rare element whose float32 and float64 sums round to neighbouring bf16
values).  Bounds: the bf16-value
regime's 2e-2, normwise and elementwise, with an elementwise floor of
5e-2 * max|ref|: such a rounding flip of one element of a bf16 operand moves
the row it feeds by one bf16 step of that element times the weights, up to
about 1e-3 of the row's largest entry when the element is among the largest
of its row (the input gradients see two such operands in a row), which
near-zero elements cannot absorb against the usual 1e-3 floor."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, bf16_round

pytestmark = pytest.mark.gpu


def _b(t: torch.Tensor) -> np.ndarray:
    """A float tensor rounded to bf16, as float64 (the operand the GPU uses)."""
    return t.detach().to(torch.bfloat16).double().cpu().numpy()


def _composition(mod, query, ref, x, shapes, starts, mask, gy):
    """Forward and backward of the layer in float64 from the oracle."""
    B, Q, C = query.shape
    S = x.shape[1]
    M, L, K = mod.n_heads, mod.n_levels, mod.n_points
    D = C // M
    P = M * L * K
    f64 = lambda t: t.detach().double().cpu().numpy()
    Wv, Wo = _b(mod.value_proj.weight), _b(mod.output_proj.weight)
    Wh = np.concatenate([_b(mod.sampling_offsets.weight), _b(mod.attention_weights.weight)], 0)
    bv, bo = f64(mod.value_proj.bias), f64(mod.output_proj.bias)
    bh = np.concatenate([f64(mod.sampling_offsets.bias), f64(mod.attention_weights.bias)], 0)
    xb, qb = _b(x), _b(query)
    sh, st = shapes.numpy(), starts.numpy()
    m = mask.numpy()
    # forward
    value = bf16_round(oracle.linear(xb, Wv, bv)).reshape(B, S, M, D)
    value[m] = 0.0
    loc, A = oracle.query_head(qb, Wh, bh, f64(ref.float()), sh, M, L, K)
    core = bf16_round(oracle.forward(value, sh, st, loc, A)).reshape(B, Q, C)
    y = oracle.linear(core, Wo, bo)
    # backward: gradient operands in bf16 (the layer's mixed precision), the
    # weight gradients rounded to bf16 as the library GEMMs return them
    g_core, g_wo, _ = oracle.linear_backward(core, Wo, bf16_round(gy))
    g_bo = gy.reshape(-1, C).sum(0)
    gv, gl, ga = oracle.backward(value, sh, st, loc, A, bf16_round(g_core).reshape(B, Q, M, D))
    gv[m] = 0.0
    gv2 = gv.reshape(B, S, C)
    g_x, g_wv, _ = oracle.linear_backward(xb, Wv, bf16_round(gv2))
    g_bv = gv2.reshape(-1, C).sum(0)
    gh, gref = oracle.query_head_backward(sh, A, gl, ga)
    g_q, g_wh, _ = oracle.linear_backward(qb, Wh, bf16_round(gh))
    g_bh = gh.reshape(-1, 3 * P).sum(0)
    g_wo, g_wv, g_wh = bf16_round(g_wo), bf16_round(g_wv), bf16_round(g_wh)
    return dict(y=y, g_q=g_q, g_ref=gref, g_x=g_x, g_wv=g_wv, g_bv=g_bv, g_wo=g_wo, g_bo=g_bo,
                g_woff=g_wh[:2 * P], g_wattn=g_wh[2 * P:], g_boff=g_bh[:2 * P], g_battn=g_bh[2 * P:])


@pytest.mark.parametrize("dims", [(2, 57, 64, 4, 4), (1, 300, 256, 8, 4)],
                         ids=["small_C64", "detr_C256"])
def test_layer_matches_float64_composition(dims):
    B, Q, C, M, K = dims
    torch.manual_seed(0)
    levels = [(16, 20), (8, 10), (4, 5), (2, 3)]
    shapes = torch.tensor(levels, dtype=torch.int64)
    starts = torch.from_numpy(wl.level_start_index(levels))
    S = int(sum(h * w for h, w in levels))
    mod = msda.MSDeformAttn(d_model=C, n_levels=4, n_heads=M, n_points=K)
    with torch.no_grad():  # offsets away from zero so that sampling moves
        mod.sampling_offsets.weight.normal_(0.0, 0.05)
        mod.sampling_offsets.bias.normal_(0.0, 1.0)
        mod.value_proj.bias.normal_(0.0, 0.1)
        mod.output_proj.bias.normal_(0.0, 0.1)
    query = torch.randn(B, Q, C)
    ref = torch.rand(B, Q, 2)
    x = torch.randn(B, S, C)
    mask = torch.zeros(B, S, dtype=torch.bool)
    mask[-1, -7:] = True
    gy = torch.randn(B, Q, C)

    want = _composition(mod, query, ref, x, shapes, starts, mask, gy.double().numpy())

    mod = mod.cuda()
    qd = query.cuda().requires_grad_(True)
    rd = ref.cuda().requires_grad_(True)
    xd = x.cuda().requires_grad_(True)
    y = mod(qd, rd, xd, shapes.cuda(), starts.cuda(), mask.cuda())
    (y * gy.cuda()).sum().backward()
    assert msda.device_status() == 0

    tol = TOL["bf16"]
    P = M * 4 * K
    got = dict(y=y, g_q=qd.grad, g_ref=rd.grad, g_x=xd.grad, g_wv=mod.value_proj.weight.grad,
               g_bv=mod.value_proj.bias.grad, g_wo=mod.output_proj.weight.grad,
               g_bo=mod.output_proj.bias.grad, g_woff=mod.sampling_offsets.weight.grad,
               g_wattn=mod.attention_weights.weight.grad, g_boff=mod.sampling_offsets.bias.grad,
               g_battn=mod.attention_weights.bias.grad)
    for k, v in got.items():
        assert_close(v, want[k], tol, f"layer {k}", elem_tol=tol, floor=5e-2)
    assert want["g_woff"].shape == (2 * P, C)
    # padded keys carry no value: their input rows get no gradient
    assert not xd.grad[-1, -7:].any()


def test_forward_uses_no_torch_linear(monkeypatch):
    """The CUDA path of the layer calls the library's dense layers, not
    torch.nn.functional.linear."""
    def boom(*a, **k):
        raise AssertionError("torch linear called on the layer's CUDA path")
    monkeypatch.setattr(torch.nn.functional, "linear", boom)
    mod = msda.MSDeformAttn(d_model=64, n_levels=2, n_heads=2, n_points=8).cuda()
    levels = torch.tensor([[8, 8], [4, 4]], dtype=torch.int64, device="cuda")
    starts = torch.tensor([0, 64], dtype=torch.int64, device="cuda")
    y = mod(torch.randn(1, 10, 64, device="cuda"), torch.rand(1, 10, 2, device="cuda"),
            torch.randn(1, 80, 64, device="cuda"), levels, starts)
    assert y.shape == (1, 10, 64) and torch.isfinite(y).all()
