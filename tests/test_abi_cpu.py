"""The C-ABI library on a machine without a GPU: it loads, exports every
function include/msda.h declares, and its host-side argument checks reject bad
calls before any CUDA call is made (no compute happens here)."""
import ctypes

import pytest

from scale_deformable_attention_msdeformattn_b200 import _lib


@pytest.fixture(scope="module")
def lib():
    from scale_deformable_attention_msdeformattn_b200 import build
    build.build()
    return _lib.load()


def test_exports_every_declared_symbol(lib):
    names = _lib.declared_functions()
    assert {"msda_forward", "msda_backward", "msda_fused_forward", "msda_fused_backward",
            "msda_zero_grads", "msda_backward_workspace_size", "msda_get_device_status",
            "msda_status_string", "msda_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert set(_lib._SIGNATURES) >= set(names)


def test_version_and_status_strings(lib):
    assert lib.msda_version().decode() == "0.1.0"
    for code in range(7):
        assert lib.msda_status_string(code)
    assert b"unknown" in lib.msda_status_string(99)


FAKE = ctypes.c_void_p(0x100000)       # 16-byte aligned, never dereferenced
MISALIGNED = ctypes.c_void_p(0x100004)


def _prob(**kw):
    d = dict(batch=1, num_keys=80, num_queries=16, num_heads=2, head_dim=8, num_levels=2,
             num_points=2, value_dtype=_lib.MSDA_F32, flags=0)
    d.update(kw)
    return _lib.Problem(**d)


def _fwd(lib, prob, **ptrs):
    p = dict(value=FAKE, shapes=FAKE, starts=FAKE, loc=FAKE, attn=FAKE, out=FAKE)
    p.update(ptrs)
    return lib.msda_forward(ctypes.byref(prob) if prob is not None else None, p["value"],
                            p["shapes"], p["starts"], p["loc"], p["attn"], p["out"], None)


@pytest.mark.parametrize("bad,code", [
    (dict(head_dim=24), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(head_dim=512), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(num_levels=17), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(num_points=33), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(num_levels=16, num_points=9), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(num_keys=1 << 27), _lib.MSDA_ERR_UNSUPPORTED),
    (dict(num_keys=0), _lib.MSDA_ERR_INVALID_ARG),
    (dict(num_heads=0), _lib.MSDA_ERR_INVALID_ARG),
    (dict(batch=-1), _lib.MSDA_ERR_INVALID_ARG),
    (dict(num_queries=-3), _lib.MSDA_ERR_INVALID_ARG),
    (dict(value_dtype=7), _lib.MSDA_ERR_INVALID_ARG),
    (dict(flags=1 << 5), _lib.MSDA_ERR_INVALID_ARG),
    (dict(flags=_lib.MSDA_GRAD_VALUE_BF16 | _lib.MSDA_ACCUMULATE_GRADS), _lib.MSDA_ERR_INVALID_ARG),
])
def test_problem_checks(lib, bad, code):
    assert _fwd(lib, _prob(**bad)) == code


def test_pointer_checks(lib):
    assert _fwd(lib, None) == _lib.MSDA_ERR_INVALID_ARG
    for k in ("value", "shapes", "starts", "loc", "attn", "out"):
        assert _fwd(lib, _prob(), **{k: None}) == _lib.MSDA_ERR_INVALID_ARG, k
        assert _fwd(lib, _prob(), **{k: MISALIGNED}) == _lib.MSDA_ERR_INVALID_ARG, k


def test_backward_checks(lib):
    prob = _prob(flags=_lib.MSDA_GRAD_VALUE_BF16)
    n = ctypes.c_size_t(0)
    assert lib.msda_backward_workspace_size(ctypes.byref(prob), ctypes.byref(n)) == 0
    assert n.value == 1 * 80 * 2 * 8 * 4
    prob32 = _prob()
    assert lib.msda_backward_workspace_size(ctypes.byref(prob32), ctypes.byref(n)) == 0
    assert n.value == 0
    # bf16 grad_value without a big enough workspace
    st = lib.msda_backward(ctypes.byref(prob), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           FAKE, 16, None)
    assert st == _lib.MSDA_ERR_INVALID_ARG
    st = lib.msda_fused_backward(ctypes.byref(_prob()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 None, FAKE, FAKE, FAKE, None, 0, None)
    assert st == _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_zero_grads(ctypes.byref(_prob()), None, None, None) == _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_get_device_status(None, None) == _lib.MSDA_ERR_INVALID_ARG


def test_product_path_has_no_oracle_import():
    """The package (binding + library) never imports the oracle."""
    import os
    import re
    pkg = os.path.dirname(_lib.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle", text, re.M), f
                assert "msda_oracle" not in text, f


def test_query_order_checks(lib):
    """query_order must be 4-byte aligned; B*Q must stay below 2^31; the sort's
    pointers are checked before anything is enqueued."""
    prob = _prob()
    prob.query_order = ctypes.c_void_p(0x100002)
    assert _fwd(lib, prob) == _lib.MSDA_ERR_INVALID_ARG
    assert _fwd(lib, _prob(batch=1 << 16, num_queries=1 << 15)) == _lib.MSDA_ERR_UNSUPPORTED
    p = _prob(batch=3, num_queries=10)
    assert lib.msda_sort_queries(ctypes.byref(p), FAKE, ctypes.c_void_p(0x100001), None) == \
        _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_sort_queries(ctypes.byref(p), None, FAKE, None) == _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_sort_queries(ctypes.byref(p), MISALIGNED, FAKE, None) == _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_sort_queries(None, FAKE, FAKE, None) == _lib.MSDA_ERR_INVALID_ARG
    # nothing to sort: succeeds without touching the device
    empty = _prob(batch=0)
    assert lib.msda_sort_queries(ctypes.byref(empty), None, None, None) == _lib.MSDA_OK


def test_int8_checks(lib):
    """MSDA_S8 needs a 4-byte aligned value_scale; the quantiser takes a
    float32 / bf16 source with D a multiple of 8 and 32-byte aligned codes."""
    p = _prob(value_dtype=_lib.MSDA_S8)
    assert _fwd(lib, p) == _lib.MSDA_ERR_INVALID_ARG
    p.value_scale = ctypes.c_void_p(0x100002)
    assert _fwd(lib, p) == _lib.MSDA_ERR_INVALID_ARG
    src = _prob(value_dtype=_lib.MSDA_S8)
    src.value_scale = FAKE
    assert lib.msda_quantize_value_s8(ctypes.byref(src), FAKE, FAKE, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    f32 = _prob()
    assert lib.msda_quantize_value_s8(ctypes.byref(f32), FAKE, MISALIGNED, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_quantize_value_s8(ctypes.byref(f32), FAKE, FAKE, None, None) == \
        _lib.MSDA_ERR_INVALID_ARG


def test_dcn_checks(lib):
    """msda_dcn_*: output size of the convolution grid, parameter checks and
    pointer checks before anything is enqueued."""
    def prob(**kw):
        d = dict(batch=2, height=56, width=56, groups=4, group_channels=16, kernel_h=3, kernel_w=3,
                 stride_h=1, stride_w=1, pad_h=1, pad_w=1, dilation_h=1, dilation_w=1,
                 value_dtype=_lib.MSDA_F32, flags=0)
        d.update(kw)
        return _lib.DcnProblem(**d)

    ho, wo = ctypes.c_int64(0), ctypes.c_int64(0)

    def size(p):
        st = lib.msda_dcn_output_size(ctypes.byref(p), ctypes.byref(ho), ctypes.byref(wo))
        return st, ho.value, wo.value

    assert size(prob()) == (0, 56, 56)
    assert size(prob(kernel_h=7, kernel_w=7, stride_h=2, stride_w=2, pad_h=3, pad_w=3)) == (0, 28, 28)
    assert size(prob(kernel_h=5, dilation_h=2, pad_h=0, height=9))[:2] == (0, 1)
    assert size(prob(kernel_h=5, dilation_h=3, pad_h=0, height=9))[:2] == (0, 0)  # nothing to sample
    assert size(prob(stride_w=0))[0] == _lib.MSDA_ERR_INVALID_ARG
    assert size(prob(pad_h=-1))[0] == _lib.MSDA_ERR_INVALID_ARG
    assert size(prob(kernel_w=33, pad_w=16))[0] == _lib.MSDA_ERR_UNSUPPORTED
    assert size(prob(kernel_h=17, pad_h=8))[0] == _lib.MSDA_ERR_UNSUPPORTED
    assert size(prob(group_channels=24))[0] == _lib.MSDA_ERR_UNSUPPORTED
    assert size(prob(value_dtype=_lib.MSDA_S8))[0] == _lib.MSDA_ERR_INVALID_ARG  # no value_scale
    p = prob()
    assert lib.msda_dcn_forward(ctypes.byref(p), MISALIGNED, FAKE, FAKE, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_dcn_forward(ctypes.byref(p), FAKE, FAKE, None, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    pb = prob(flags=_lib.MSDA_GRAD_VALUE_BF16)
    assert lib.msda_dcn_backward_workspace_size(ctypes.byref(pb), ctypes.byref(n)) == 0
    assert n.value == 2 * 56 * 56 * 4 * 16 * 4
    assert lib.msda_dcn_backward(ctypes.byref(pb), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                 16, None) == _lib.MSDA_ERR_INVALID_ARG


def test_fp8_checks(lib):
    """MSDA_E4M3 needs a 4-byte aligned value_scale; the FP8 quantiser takes a
    float32 / bf16 source, 32-byte aligned codes and a scale array."""
    p = _prob(value_dtype=_lib.MSDA_E4M3)
    assert _fwd(lib, p) == _lib.MSDA_ERR_INVALID_ARG
    p.value_scale = ctypes.c_void_p(0x100002)
    assert _fwd(lib, p) == _lib.MSDA_ERR_INVALID_ARG
    src = _prob(value_dtype=_lib.MSDA_E4M3)
    src.value_scale = FAKE
    assert lib.msda_quantize_value_e4m3(ctypes.byref(src), FAKE, FAKE, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    f32 = _prob()
    assert lib.msda_quantize_value_e4m3(ctypes.byref(f32), FAKE, MISALIGNED, FAKE, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    assert lib.msda_quantize_value_e4m3(ctypes.byref(f32), FAKE, FAKE, None, None) == \
        _lib.MSDA_ERR_INVALID_ARG
    empty = _prob(batch=0)
    assert lib.msda_quantize_value_e4m3(ctypes.byref(empty), None, None, None, None) == _lib.MSDA_OK


def test_dense_layer_checks(lib):
    """msda_linear, msda_query_head and msda_query_head_backward reject bad
    sizes and pointers before anything is enqueued; empty inputs are a no-op."""
    F32, BF16 = _lib.MSDA_F32, _lib.MSDA_BF16
    bad, unsupported, ok = _lib.MSDA_ERR_INVALID_ARG, _lib.MSDA_ERR_UNSUPPORTED, _lib.MSDA_OK

    def linear(rows=100, k=16, n=16, x=FAKE, w=FAKE, b=None, out=FAKE, dt=F32):
        return lib.msda_linear(rows, k, n, x, w, b, out, dt, None)

    assert linear(k=12) == bad                        # in_features a multiple of 8
    assert linear(k=0) == bad
    assert linear(n=20) == bad                        # out_features a multiple of 8
    assert linear(dt=_lib.MSDA_S8) == bad             # float32 or bf16 output only
    assert linear(rows=-1) == bad
    assert linear(rows=0, x=None, w=None, out=None) == ok
    assert linear(x=MISALIGNED) == bad
    assert linear(out=None, dt=BF16) == bad
    assert linear(b=ctypes.c_void_p(0x100002)) == bad  # bias 4-byte aligned

    def head(p, k=256, q=FAKE, ref=FAKE, loc=FAKE, attn=FAKE):
        return lib.msda_query_head(ctypes.byref(p), k, q, FAKE, None, ref, FAKE, loc, attn, None)

    def head_bwd(p, gh=FAKE):
        return lib.msda_query_head_backward(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, gh, None, None)

    good = _prob(num_heads=8, num_levels=4, num_points=4)          # L*K = 16, P = 128
    assert head(good, k=12) == bad
    assert head(good, q=MISALIGNED) == bad
    assert head(good, loc=None) == bad
    assert head_bwd(good, gh=MISALIGNED) == bad
    # L*K a power of two of at most 32, M*L*K a multiple of 32
    for p in (_prob(num_heads=32, num_levels=3, num_points=1), _prob(num_heads=1, num_levels=2, num_points=2),
              _prob(num_heads=1, num_levels=4, num_points=16)):
        assert head(p) == unsupported
        assert head_bwd(p) == unsupported
    empty = _prob(batch=0, num_heads=8, num_levels=4, num_points=4)
    assert head(empty, q=None, ref=None, loc=None, attn=None) == ok
    assert head_bwd(empty, gh=None) == ok
