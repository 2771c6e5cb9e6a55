"""Tensor-core dense layers (msda_linear, msda_query_head,
msda_query_head_backward) against the fp64 oracle on the same seeded,
bf16-exact inputs.  Needs a B200 (sm_100a).

The products of bf16 operands are exact in float32, so the only difference
from the oracle's float64 sums is the float32 accumulation order: float32
outputs are held to the float32 bounds of the operator's tests (1e-5
normwise, 1e-3 elementwise with the 1e-3 * max floor), bf16 outputs to one
bf16 step (2^-7 of the value) against the oracle rounded to bf16."""
import numpy as np
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, bf16_round

pytestmark = pytest.mark.gpu


def _bf16(seed, tag, shape, scale=1.0):
    """Seeded normal draws rounded to bf16: (device tensor, exact float64)."""
    n = int(np.prod(shape))
    bits = wl.to_bf16_bits(scale * wl.normal(seed, tag, n)).reshape(shape)
    t = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return t, wl.bf16_bits_to_f64(bits)


def _f32(seed, tag, shape, scale=1.0, uniform=False):
    n = int(np.prod(shape))
    x = (wl.uniform(seed, tag, n) if uniform else scale * wl.normal(seed, tag, n)).astype(np.float32)
    x = x.reshape(shape)
    return torch.from_numpy(x).cuda(), x.astype(np.float64)


LINEAR = [
    # rows, in_features, out_features, bias, out dtype
    (1, 8, 8, False, "f32"),
    (100, 64, 104, True, "f32"),
    (128, 256, 128, True, "f32"),
    (129, 72, 256, False, "f32"),
    (777, 256, 384, True, "f32"),
    (300, 136, 600, True, "f32"),
    (4099, 256, 256, True, "bf16"),
    (255, 64, 40, False, "bf16"),
    # w too large to stay in shared memory (more than 4 K blocks at 256
    # output columns, more than 8 at 128): w streams through the ring with x
    (513, 320, 256, True, "f32"),
    (1000, 384, 256, False, "f32"),
    (300, 576, 104, True, "bf16"),
]


@pytest.mark.parametrize("spec", LINEAR, ids=[f"{r}x{k}x{n}_{'b' if b else 'nb'}_{o}" for r, k, n, b, o in LINEAR])
def test_linear_matches_oracle(spec):
    rows, K, N, with_bias, out = spec
    seed = 0x5EED0100 + rows + K + N
    x, x64 = _bf16(seed, 1, (rows, K))
    w, w64 = _bf16(seed, 2, (N, K), scale=K ** -0.5)
    b, b64 = _f32(seed, 3, (N,)) if with_bias else (None, None)
    y = msda.linear(x, w, b, out_dtype=torch.float32 if out == "f32" else torch.bfloat16)
    assert msda.device_status() == 0
    ref = oracle.linear(x64, w64, b64)
    if out == "f32":
        assert_close(y, ref, TOL["f32"], f"linear {spec}")
    else:
        assert_close(y, bf16_round(ref), 2.0 ** -7, f"linear {spec} vs rounded oracle", elem_tol=2.0 ** -7)


def test_value_projection_writes_the_operator_layout():
    """value_proj with a bf16 output of M*D features is the operator's value
    tensor [B, S, M, D]: the core run on it equals the oracle core run on the
    oracle's projection (rounded to bf16 the same way)."""
    B, S, C, M, D = 2, 80, 64, 2, 32
    seed = 0x5EED0200
    xin, x64 = _bf16(seed, 1, (B, S, C))
    w, w64 = _bf16(seed, 2, (M * D, C), scale=C ** -0.5)
    v = msda.linear(xin, w, out_dtype=torch.bfloat16).view(B, S, M, D)
    ref = bf16_round(oracle.linear(x64, w64)).reshape(B, S, M, D)
    assert_close(v, ref, 2.0 ** -7, "value_proj", elem_tol=2.0 ** -7)


HEAD = [
    # B, Q, C, M, levels, K, offset scale (pixels)
    (2, 301, 256, 8, [(20, 30), (10, 15), (5, 8), (3, 4)], 4, 2.0),
    (1, 130, 64, 1, [(16, 16), (8, 8), (4, 4), (2, 2)], 8, 3.0),
    (3, 64, 128, 2, [(9, 13), (5, 7), (3, 4), (2, 2)], 4, 1.0),
]


def _head_inputs(spec, seed):
    B, Q, C, M, levels, K, sig = spec
    L = len(levels)
    P = M * L * K
    q, q64 = _bf16(seed, 1, (B, Q, C))
    w, w64 = _bf16(seed, 2, (3 * P, C), scale=C ** -0.5)
    b, b64 = _f32(seed, 3, (3 * P,), scale=0.5)
    # offsets of about `sig` level pixels, logits of about 1
    w64 = w64.copy()
    scale = np.ones(3 * P)
    scale[:2 * P] = sig
    wb = wl.to_bf16_bits(w64 * scale[:, None]).reshape(3 * P, C)
    w = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    w64 = wl.bf16_bits_to_f64(wb)
    ref, ref64 = _f32(seed, 4, (B, Q, 2), uniform=True)
    shapes = np.array(levels, np.int64)
    return q, q64, w, w64, b, b64, ref, ref64, shapes


@pytest.mark.parametrize("spec", HEAD, ids=["detr_like", "k8_one_head", "small"])
def test_query_head_matches_oracle(spec):
    B, Q, C, M, levels, K, sig = spec
    q, q64, w, w64, b, b64, ref, ref64, shapes = _head_inputs(spec, 0x5EED0300 + Q)
    loc, attn = msda.query_head(q, w, b, ref, torch.from_numpy(shapes).cuda(), M, K)
    assert msda.device_status() == 0
    r_loc, r_attn = oracle.query_head(q64, w64, b64, ref64, shapes, M, len(levels), K)
    assert_close(loc, r_loc, TOL["f32"], f"query head locations {spec[:2]}")
    assert_close(attn, r_attn, TOL["f32"], f"query head attention weights {spec[:2]}")


@pytest.mark.parametrize("spec", HEAD, ids=["detr_like", "k8_one_head", "small"])
def test_query_head_backward_matches_oracle(spec):
    B, Q, C, M, levels, K, sig = spec
    L = len(levels)
    seed = 0x5EED0400 + Q
    q, q64, w, w64, b, b64, ref, ref64, shapes = _head_inputs(spec, seed)
    _, r_attn = oracle.query_head(q64, w64, b64, ref64, shapes, M, L, K)
    a = torch.from_numpy(r_attn.astype(np.float32)).cuda()
    a64 = a.double().cpu().numpy()
    gl, gl64 = _f32(seed, 5, (B, Q, M, L, K, 2))
    ga, ga64 = _f32(seed, 6, (B, Q, M, L, K))
    gh, gref = msda.query_head_backward(a, gl, ga, torch.from_numpy(shapes).cuda(),
                                        want_grad_reference_points=True)
    assert msda.device_status() == 0
    r_gh, r_gref = oracle.query_head_backward(shapes, a64, gl64, ga64)
    assert_close(gh, r_gh, TOL["f32"], "query head grad")
    assert_close(gref, r_gref, TOL["f32"], "query head grad_reference_points")


def test_query_head_rejects_unsupported_sizes():
    """L*K must be a power of two of at most 32 and M*L*K a multiple of 32."""
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    for M, levels, K in [(1, [(4, 4)], 3), (2, [(4, 4), (2, 2)], 2), (1, [(4, 4)] * 4, 16)]:
        L = len(levels)
        P = M * L * K
        w = torch.zeros((3 * P, 64), dtype=torch.bfloat16, device="cuda")
        ref = torch.zeros((1, 4, 2), device="cuda")
        sh = torch.tensor(levels, dtype=torch.int64, device="cuda")
        with pytest.raises(msda.MsdaError) as e:
            msda.query_head(q, w, None, ref, sh, M, K)
        assert e.value.status == 2


def test_gemm_bounded_waits_report_timeout_and_context_survives():
    """With MSDA_TEST_WITHHOLD_COPY the query head's tensor-core kernel arms
    each CTA's first operand stage without loading it: the MMA lane's wait
    and the producer's waits run out (about a second each), the kernel
    reports MSDA_ERR_DEVICE_TIMEOUT, frees its tensor memory and returns,
    and the next calls (query head and plain dense layer) are correct."""
    import ctypes
    from scale_deformable_attention_msdeformattn_b200 import _lib
    spec = HEAD[0]
    B, Q, C, M, levels, K, sig = spec
    L = len(levels)
    P = M * L * K
    q, q64, w, w64, b, b64, ref, ref64, shapes = _head_inputs(spec, 0x5EED0500)
    sh = torch.from_numpy(shapes).cuda()
    loc = torch.empty((B, Q, M, L, K, 2), device="cuda")
    attn = torch.empty((B, Q, M, L, K), device="cuda")
    prob = _lib.Problem(B, 1, Q, M, 8, L, K, _lib.MSDA_F32, _lib.MSDA_TEST_WITHHOLD_COPY)
    p = lambda z: ctypes.c_void_p(z.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert msda.device_status() == 0
    st = _lib.load().msda_query_head(ctypes.byref(prob), C, p(q), p(w), p(b), p(ref), p(sh), p(loc),
                                     p(attn), stream)
    assert st == 0
    assert msda.device_status() == _lib.MSDA_ERR_DEVICE_TIMEOUT
    # the context is intact and the kernel's tensor memory was freed
    loc2, attn2 = msda.query_head(q, w, b, ref, sh, M, K)
    assert msda.device_status() == 0
    r_loc, r_attn = oracle.query_head(q64, w64, b64, ref64, shapes, M, L, K)
    assert_close(loc2, r_loc, TOL["f32"], "query head after a time-out")
    assert_close(attn2, r_attn, TOL["f32"], "attention weights after a time-out")
    x, x64 = _bf16(0x5EED0501, 1, (1000, 256))
    wt, wt64 = _bf16(0x5EED0501, 2, (256, 256), scale=256 ** -0.5)
    y = msda.linear(x, wt, None, out_dtype=torch.float32)
    assert msda.device_status() == 0
    assert_close(y, oracle.linear(x64, wt64), TOL["f32"], "linear after a time-out")
