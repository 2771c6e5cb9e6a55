"""msda_backward_noalloc: the backward for callers that cannot allocate.

Some callers cannot allocate device memory when they run the backward pass: a
host framework that hands an extension only its input and output tensors and
no workspace, or a serving process whose device memory is fixed once it has
started.  msda_backward_noalloc serves them by summing into a float32 buffer
the library owns.  These tests call it through the C ABI and compare it with
msda_backward given a caller workspace (the existing path), on two calls in a
row, so that a buffer left dirty by the first call would show up in the
second, and with the fp64 oracle (grad_value against the oracle's rounded to
bf16, the other gradients at the workload's tolerance, both metrics).  This
file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from scale_deformable_attention_msdeformattn_b200 import _lib
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, bf16_round, oracle_nonfused, rel_err, upload

pytestmark = pytest.mark.gpu

SCRATCH_FLOATS = 4 << 20  # the library's buffer: 4 Mi float32


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _problem(w: wl.Workload, flags: int) -> _lib.Problem:
    dt = _lib.MSDA_BF16 if w.dtype == "bf16" else _lib.MSDA_F32
    return _lib.Problem(w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K, dt, flags)


def _outputs(w: wl.Workload, dev):
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    gv = torch.full((B, S, M, D), float("nan"), dtype=torch.bfloat16, device=dev)
    gl = torch.full((B, Q, M, L, K, 2), float("nan"), dtype=torch.float32, device=dev)
    ga = torch.full((B, Q, M, L, K), float("nan"), dtype=torch.float32, device=dev)
    return gv, gl, ga


@pytest.mark.parametrize("spec", [
    ("noalloc_bf16", 2, [(20, 30), (10, 15), (5, 8)], 57, 4, 32, 4, "bf16", 2.0),
    ("noalloc_f32", 1, [(40, 60), (20, 30)], 133, 8, 32, 4, "f32", 3.0),
])
def test_noalloc_matches_workspace_backward(spec):
    name, B, levels, Q, M, D, K, dtype, sigma = spec
    w = wl.custom(name, B, levels, Q, M, D, K, dtype, "uniform", sigma, index=400)
    assert w.B * w.S * w.M * w.D <= SCRATCH_FLOATS
    x = wl.generate(w)
    t = upload(x)
    dev = t["value"].device
    lib = _lib.load()
    prob = _problem(w, _lib.MSDA_GRAD_VALUE_BF16)
    args = (_p(t["value"]), _p(t["spatial_shapes"]), _p(t["level_start_index"]),
            _p(t["sampling_locations"]), _p(t["attention_weights"]), _p(t["grad_output"]))

    # existing path: msda_backward with a caller-provided workspace
    nbytes = ctypes.c_size_t(0)
    assert lib.msda_backward_workspace_size(ctypes.byref(prob), ctypes.byref(nbytes)) == 0
    ws = torch.empty(nbytes.value, dtype=torch.uint8, device=dev)
    ref_gv, ref_gl, ref_ga = _outputs(w, dev)
    st = lib.msda_backward(ctypes.byref(prob), *args, _p(ref_gv), _p(ref_gl), _p(ref_ga), _p(ws),
                           nbytes.value, _stream())
    assert st == 0
    torch.cuda.synchronize()

    _, o_gv, o_gl, o_ga = oracle_nonfused(x)
    for call in range(2):
        gv, gl, ga = _outputs(w, dev)
        st = lib.msda_backward_noalloc(ctypes.byref(prob), *args, _p(gv), _p(gl), _p(ga), _stream())
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        ref = ref_gv.double().cpu().numpy()
        assert rel_err(gv, ref) <= TOL["bf16"], f"call {call}: grad_value"
        assert rel_err(gl, ref_gl.double().cpu().numpy()) <= TOL[w.dtype], f"call {call}: grad_loc"
        assert rel_err(ga, ref_ga.double().cpu().numpy()) <= TOL[w.dtype], f"call {call}: grad_attn"
        # against the oracle: grad_value is its float64 sum rounded to bf16 up
        # to one rounding step (at most 2^-7 of the value), the other
        # gradients at the workload's bounds
        assert_close(gv, bf16_round(o_gv), 2.0 ** -7, f"no-alloc call {call}: grad_value vs rounded oracle",
                     elem_tol=2.0 ** -7)
        assert_close(gl, o_gl, TOL[w.dtype], f"no-alloc call {call}: grad_loc vs oracle")
        assert_close(ga, o_ga, TOL[w.dtype], f"no-alloc call {call}: grad_attn vs oracle")

    code = ctypes.c_int32(-1)
    assert lib.msda_get_device_status(_stream(), ctypes.byref(code)) == 0 and code.value == 0


def test_noalloc_rejects_problems_beyond_its_buffer():
    """B*S*M*D above the buffer is refused before anything is enqueued."""
    lib = _lib.load()
    fake = ctypes.c_void_p(0x100000)
    prob = _lib.Problem(2, 80000, 16, 8, 32, 2, 2, _lib.MSDA_BF16, _lib.MSDA_GRAD_VALUE_BF16)
    assert prob.batch * prob.num_keys * prob.num_heads * prob.head_dim > SCRATCH_FLOATS
    st = lib.msda_backward_noalloc(ctypes.byref(prob), fake, fake, fake, fake, fake, fake, fake,
                                   fake, fake, None)
    assert st == _lib.MSDA_ERR_UNSUPPORTED
    bad_flags = _lib.Problem(1, 80, 16, 2, 8, 2, 2, _lib.MSDA_F32, _lib.MSDA_ACCUMULATE_GRADS)
    st = lib.msda_backward_noalloc(ctypes.byref(bad_flags), fake, fake, fake, fake, fake, fake, fake,
                                   fake, fake, None)
    assert st == _lib.MSDA_ERR_INVALID_ARG
