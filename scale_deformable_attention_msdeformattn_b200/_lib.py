"""ctypes view of libmsda.so (include/msda.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os
import re
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmsda.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "msda.h")

MSDA_OK = 0
MSDA_ERR_INVALID_ARG = 1
MSDA_ERR_UNSUPPORTED = 2
MSDA_ERR_CUDA = 3
MSDA_ERR_DEVICE_CHECK = 4
MSDA_ERR_DEVICE_TIMEOUT = 5
MSDA_ERR_DEVICE_BOUNDS = 6

MSDA_F32 = 0
MSDA_BF16 = 1
MSDA_S8 = 2
MSDA_E4M3 = 3

MSDA_GRAD_VALUE_BF16 = 1 << 0
MSDA_ACCUMULATE_GRADS = 1 << 1
MSDA_STAGE_INPUTS = 1 << 2
MSDA_MERGE_REDUCTIONS = 1 << 3
MSDA_TEST_WITHHOLD_COPY = 1 << 31


class Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("num_keys", ctypes.c_int64),
        ("num_queries", ctypes.c_int64),
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("num_levels", ctypes.c_int32),
        ("num_points", ctypes.c_int32),
        ("value_dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("query_order", ctypes.c_void_p),
        ("value_scale", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_PROB = ctypes.POINTER(Problem)
class DcnProblem(ctypes.Structure):
    """msda_dcn_problem of include/msda.h."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("height", ctypes.c_int32),
        ("width", ctypes.c_int32),
        ("groups", ctypes.c_int32),
        ("group_channels", ctypes.c_int32),
        ("kernel_h", ctypes.c_int32),
        ("kernel_w", ctypes.c_int32),
        ("stride_h", ctypes.c_int32),
        ("stride_w", ctypes.c_int32),
        ("pad_h", ctypes.c_int32),
        ("pad_w", ctypes.c_int32),
        ("dilation_h", ctypes.c_int32),
        ("dilation_w", ctypes.c_int32),
        ("value_dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("value_scale", ctypes.c_void_p),
    ]


_DCN = ctypes.POINTER(DcnProblem)

_SIGNATURES = {
    "msda_forward": [_PROB, _P, _P, _P, _P, _P, _P, _P],
    "msda_backward": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "msda_fused_forward": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "msda_fused_backward": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "msda_backward_workspace_size": [_PROB, ctypes.POINTER(ctypes.c_size_t)],
    "msda_zero_grads": [_PROB, _P, _P, _P],
    "msda_backward_noalloc": [_PROB, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P],
    "msda_sort_queries": [_PROB, _P, _P, _P],
    "msda_quantize_value_s8": [_PROB, _P, _P, _P, _P],
    "msda_quantize_value_e4m3": [_PROB, _P, _P, _P, _P],
    "msda_dcn_output_size": [_DCN, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64)],
    "msda_dcn_forward": [_DCN, _P, _P, _P, _P, _P],
    "msda_dcn_backward": [_DCN, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
    "msda_dcn_backward_workspace_size": [_DCN, ctypes.POINTER(ctypes.c_size_t)],
    "msda_linear": [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_int32, _P],
    "msda_query_head": [_PROB, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P],
    "msda_query_head_backward": [_PROB, _P, _P, _P, _P, _P, _P, _P],
    "msda_get_device_status": [_P, ctypes.POINTER(ctypes.c_int32)],
    "msda_status_string": [ctypes.c_int],
    "msda_version": [],
}

_lib = None
_lock = threading.Lock()


def declared_functions(header: str = HEADER):
    """Names of the functions include/msda.h declares."""
    text = open(header).read()
    return sorted(set(re.findall(r"^\s*MSDA_API\s+(?:const\s+)?[a-z_]+\s*\*?\s*(msda_[a-z_0-9]+)\s*\(", text, re.M)))


def load(path: str = LIB_PATH):
    """Loads libmsda.so; raises if it was not built (there is no fallback)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                "libmsda.so is missing (%s): build it with "
                "`python -m scale_deformable_attention_msdeformattn_b200.build`" % path)
        lib = ctypes.CDLL(path)
        for name, args in _SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.msda_status_string.restype = ctypes.c_char_p
        lib.msda_version.restype = ctypes.c_char_p
        _lib = lib
        return lib
