"""fp64 CPU oracle for multi-scale deformable attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

The arithmetic lives in ``msda_oracle.c`` (plain C, double precision, direct
loops over the defining sums); this module only compiles it with gcc, widens
inputs to float64 and passes pointers.  See the C file's header for the page
citations and the readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libmsda_oracle.so")
_lib = None
_lock = threading.Lock()


class _Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("B", "S", "Q", "M", "D", "L", "K")]


class _DcnDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("N", "H", "W", "G", "C", "Ho", "Wo", "kh", "kw",
                                              "stride_h", "stride_w", "pad_h", "pad_w",
                                              "dil_h", "dil_w")]


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc into oracle/_build (no GPU involved)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            D = ctypes.POINTER(_Dims)
            lib.msda_oracle_forward.argtypes = [D, P, P, P, P, P, P]
            lib.msda_oracle_backward.argtypes = [D, P, P, P, P, P, P, P, P, P]
            lib.msda_oracle_sampling_locations.argtypes = [D, P, P, P, P]
            lib.msda_oracle_softmax.argtypes = [D, P, P]
            lib.msda_oracle_fused_chain.argtypes = [D, P, P, P, P, P, P, P]
            lib.msda_oracle_quantize_value_s8.argtypes = [D, P, P, P]
            lib.msda_oracle_quantize_value_e4m3.argtypes = [D, P, P, P]
            lib.msda_oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.msda_oracle_e4m3_encode.restype = ctypes.c_ubyte
            lib.msda_oracle_e4m3_decode.argtypes = [ctypes.c_ubyte]
            lib.msda_oracle_e4m3_decode.restype = ctypes.c_double
            DD = ctypes.POINTER(_DcnDims)
            lib.msda_oracle_dcn_forward.argtypes = [DD, P, P, P, P]
            lib.msda_oracle_dcn_backward.argtypes = [DD, P, P, P, P, P, P, P]
            I = ctypes.c_int64
            lib.msda_oracle_linear.argtypes = [I, I, I, P, P, P, P]
            lib.msda_oracle_linear_backward.argtypes = [I, I, I, P, P, P, P, P, P]
            for f in ("msda_oracle_forward", "msda_oracle_backward", "msda_oracle_sampling_locations",
                      "msda_oracle_softmax", "msda_oracle_fused_chain",
                      "msda_oracle_quantize_value_s8", "msda_oracle_quantize_value_e4m3",
                      "msda_oracle_dcn_forward",
                      "msda_oracle_dcn_backward", "msda_oracle_linear",
                      "msda_oracle_linear_backward"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(value: np.ndarray, loc_like: np.ndarray) -> _Dims:
    B, S, M, D = value.shape
    _, Q, M2, L, K = loc_like.shape[:5]
    assert M2 == M and loc_like.shape[0] == B
    return _Dims(B, S, Q, M, D, L, K)


def forward(value, spatial_shapes, level_start_index, sampling_locations, attention_weights):
    """out[B,Q,M,D] (float64) of the core operator."""
    v, sh, st = _f64(value), _i64(spatial_shapes), _i64(level_start_index)
    loc, a = _f64(sampling_locations), _f64(attention_weights)
    d = _dims(v, a)
    out = np.empty((d.B, d.Q, d.M, d.D), np.float64)
    _load().msda_oracle_forward(ctypes.byref(d), _p(v), _p(sh), _p(st), _p(loc), _p(a), _p(out))
    return out


def backward(value, spatial_shapes, level_start_index, sampling_locations, attention_weights,
             grad_output):
    """(grad_value [B,S,M,D], grad_sampling_locations [B,Q,M,L,K,2],
    grad_attention_weights [B,Q,M,L,K]), float64."""
    v, sh, st = _f64(value), _i64(spatial_shapes), _i64(level_start_index)
    loc, a, g = _f64(sampling_locations), _f64(attention_weights), _f64(grad_output)
    d = _dims(v, a)
    gv = np.empty_like(v)
    gl = np.empty_like(loc)
    ga = np.empty_like(a)
    _load().msda_oracle_backward(ctypes.byref(d), _p(v), _p(sh), _p(st), _p(loc), _p(a), _p(g),
                                 _p(gv), _p(gl), _p(ga))
    return gv, gl, ga


def sampling_locations(spatial_shapes, reference_points, sampling_offsets):
    """loc = ref + off / (W_l, H_l), float64 [B,Q,M,L,K,2]."""
    sh, ref, off = _i64(spatial_shapes), _f64(reference_points), _f64(sampling_offsets)
    B, Q, M, L, K, _ = off.shape
    d = _Dims(B, 0, Q, M, 0, L, K)
    loc = np.empty_like(off)
    _load().msda_oracle_sampling_locations(ctypes.byref(d), _p(sh), _p(ref), _p(off), _p(loc))
    return loc


def softmax(attention_logits, L: int, K: int):
    """Softmax over the L*K logits of each (b,q,m); returns [B,Q,M,L,K] float64."""
    z = _f64(attention_logits)
    B, Q, M, n = z.shape
    assert n == L * K
    d = _Dims(B, 0, Q, M, 0, L, K)
    a = np.empty_like(z)
    _load().msda_oracle_softmax(ctypes.byref(d), _p(z), _p(a))
    return a.reshape(B, Q, M, L, K)


def fused_chain(spatial_shapes, attention_weights, grad_loc, grad_attn, want_ref: bool = True):
    """(grad_offsets, grad_reference_points or None, grad_logits)."""
    sh, a, gl, ga = _i64(spatial_shapes), _f64(attention_weights), _f64(grad_loc), _f64(grad_attn)
    B, Q, M, L, K = a.shape
    d = _Dims(B, 0, Q, M, 0, L, K)
    goff = np.empty_like(gl)
    gref = np.empty((B, Q, 2), np.float64) if want_ref else None
    glog = np.empty((B, Q, M, L * K), np.float64)
    _load().msda_oracle_fused_chain(ctypes.byref(d), _p(sh), _p(a), _p(gl), _p(ga), _p(goff),
                                    _p(gref) if want_ref else None, _p(glog))
    return goff, gref, glog


def fused_forward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                  attention_logits):
    """Fused forward: locations and softmax first, then the core sum.

    Returns (out, attention_weights, sampling_locations), float64."""
    loc = sampling_locations(spatial_shapes, reference_points, sampling_offsets)
    L, K = loc.shape[3], loc.shape[4]
    a = softmax(attention_logits, L, K)
    return forward(value, spatial_shapes, level_start_index, loc, a), a, loc


def fused_backward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                   attention_logits, grad_output, want_ref: bool = True):
    """(grad_value, grad_reference_points, grad_sampling_offsets, grad_attention_logits)."""
    loc = sampling_locations(spatial_shapes, reference_points, sampling_offsets)
    L, K = loc.shape[3], loc.shape[4]
    a = softmax(attention_logits, L, K)
    gv, gl, ga = backward(value, spatial_shapes, level_start_index, loc, a, grad_output)
    goff, gref, glog = fused_chain(spatial_shapes, a, gl, ga, want_ref)
    return gv, gref, goff, glog


def pixel_coordinates(spatial_shapes, sampling_locations):
    """fp64 pixel coordinates (x, y) = (loc_x*W - 0.5, loc_y*H - 0.5) of each
    sample; tests use them to find samples that sit on a cell edge."""
    sh = _i64(spatial_shapes)
    loc = _f64(sampling_locations)
    W = sh[:, 1].astype(np.float64)[None, None, None, :, None]
    H = sh[:, 0].astype(np.float64)[None, None, None, :, None]
    return loc[..., 0] * W - 0.5, loc[..., 1] * H - 0.5


def quantize_value_s8(value):
    """INT8 value storage: (q int8 [B,S,M,D], scale float32 [B,M]) with one
    symmetric absmax scale per (batch, head).  `value` is float32, or bfloat16
    bit patterns (uint16), widened exactly to float32."""
    v = np.asarray(value)
    if v.dtype == np.uint16:
        v = (v.astype(np.uint32) << np.uint32(16)).view(np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    B, S, M, D = v.shape
    d = _Dims(B, S, 0, M, D, 0, 0)
    q = np.empty(v.shape, np.int8)
    scale = np.empty((B, M), np.float32)
    _load().msda_oracle_quantize_value_s8(ctypes.byref(d), _p(v), _p(q), _p(scale))
    return q, scale


def dequantize_value_s8(q, scale):
    """q * scale in float64 (exact), [B,S,M,D]: the value the operator samples."""
    return np.asarray(q, np.float64) * np.asarray(scale, np.float64)[:, None, :, None]


def e4m3_encode(x) -> np.ndarray:
    """E4M3 codes (uint8) of float32 values (finite), elementwise: the
    nearest representable value, ties to the even mantissa, clipped to +-448."""
    lib = _load()
    x = np.asarray(x, np.float32)
    return np.array([lib.msda_oracle_e4m3_encode(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


_e4m3_table = None


def e4m3_decode(c) -> np.ndarray:
    """The float64 values of E4M3 codes (NaN codes give NaN)."""
    global _e4m3_table
    if _e4m3_table is None:
        lib = _load()
        _e4m3_table = np.array([lib.msda_oracle_e4m3_decode(i) for i in range(256)], np.float64)
    return _e4m3_table[np.asarray(c, np.uint8)]


def quantize_value_e4m3(value):
    """FP8 (E4M3) value storage: (codes uint8 [B,S,M,D], scale float32 [B,M])
    with one absmax scale per (batch, head), amax / 448.  `value` is float32,
    or bfloat16 bit patterns (uint16), widened exactly to float32."""
    v = np.asarray(value)
    if v.dtype == np.uint16:
        v = (v.astype(np.uint32) << np.uint32(16)).view(np.float32)
    v = np.ascontiguousarray(v, dtype=np.float32)
    B, S, M, D = v.shape
    d = _Dims(B, S, 0, M, D, 0, 0)
    q = np.empty(v.shape, np.uint8)
    scale = np.empty((B, M), np.float32)
    _load().msda_oracle_quantize_value_e4m3(ctypes.byref(d), _p(v), _p(q), _p(scale))
    return q, scale


def dequantize_value_e4m3(q, scale):
    """decode(q) * scale in float64 (exact), [B,S,M,D]: the value the operator
    samples."""
    return e4m3_decode(q) * np.asarray(scale, np.float64)[:, None, :, None]


def dcn_output_size(H: int, W: int, kernel, stride=(1, 1), pad=(0, 0), dil=(1, 1)):
    """(Ho, Wo) of the convolution grid."""
    kh, kw = kernel
    return ((H + 2 * pad[0] - dil[0] * (kh - 1) - 1) // stride[0] + 1,
            (W + 2 * pad[1] - dil[1] * (kw - 1) - 1) // stride[1] + 1)


def _dcn_dims(x, kernel, stride, pad, dil):
    N, H, W, G, C = x.shape
    Ho, Wo = dcn_output_size(H, W, kernel, stride, pad, dil)
    return _DcnDims(N, H, W, G, C, Ho, Wo, kernel[0], kernel[1], stride[0], stride[1],
                    pad[0], pad[1], dil[0], dil[1])


def dcn_forward(x, offset, mask, kernel, stride=(1, 1), pad=(0, 0), dil=(1, 1)):
    """DCNv3 core forward, float64: x [N,H,W,G,C], offset [N,Ho,Wo,G,K,2]
    (x, y) pixels, mask [N,Ho,Wo,G,K] -> y [N,Ho,Wo,G,C]."""
    xv, off, m = _f64(x), _f64(offset), _f64(mask)
    d = _dcn_dims(xv, kernel, stride, pad, dil)
    assert off.shape == (d.N, d.Ho, d.Wo, d.G, d.kh * d.kw, 2) and m.shape == off.shape[:-1]
    y = np.empty((d.N, d.Ho, d.Wo, d.G, d.C), np.float64)
    _load().msda_oracle_dcn_forward(ctypes.byref(d), _p(xv), _p(off), _p(m), _p(y))
    return y


def dcn_backward(x, offset, mask, grad_y, kernel, stride=(1, 1), pad=(0, 0), dil=(1, 1)):
    """(grad_x, grad_offset, grad_mask), float64."""
    xv, off, m, gy = _f64(x), _f64(offset), _f64(mask), _f64(grad_y)
    d = _dcn_dims(xv, kernel, stride, pad, dil)
    assert gy.shape == (d.N, d.Ho, d.Wo, d.G, d.C)
    gx = np.empty_like(xv)
    goff = np.empty_like(off)
    gm = np.empty_like(m)
    _load().msda_oracle_dcn_backward(ctypes.byref(d), _p(xv), _p(off), _p(m), _p(gy), _p(gx),
                                     _p(goff), _p(gm))
    return gx, goff, gm


# ------------------------------------------------ the module's dense layers --

def linear(x, weight, bias=None):
    """y = x @ weight^T + bias in float64 (nn.Linear's convention): x [..., K],
    weight [N, K], bias [N] or None; returns [..., N].  The module's value and
    output projections and its query head (discosf.com §2.2, §3.1;
    cf-1.com §3.2)."""
    x, w = _f64(x), _f64(weight)
    K = x.shape[-1]
    N = w.shape[0]
    assert w.shape == (N, K)
    rows = int(np.prod(x.shape[:-1]))
    b = _f64(bias) if bias is not None else None
    y = np.empty(x.shape[:-1] + (N,), np.float64)
    _load().msda_oracle_linear(rows, K, N, _p(x), _p(w), _p(b) if b is not None else None, _p(y))
    return y


def linear_backward(x, weight, grad_y):
    """(grad_x, grad_weight, grad_bias) of linear() for an upstream grad_y."""
    x, w, gy = _f64(x), _f64(weight), _f64(grad_y)
    K, N = x.shape[-1], w.shape[0]
    rows = int(np.prod(x.shape[:-1]))
    gx = np.empty_like(x)
    gw = np.empty((N, K), np.float64)
    gb = np.empty(N, np.float64)
    _load().msda_oracle_linear_backward(rows, K, N, _p(x), _p(w), _p(gy), _p(gx), _p(gw), _p(gb))
    return gx, gw, gb


def query_head(query, weight, bias, reference_points, spatial_shapes, M: int, L: int, K: int):
    """The query head as the pages compose it (cf-1.com §3.2): one linear
    layer to 3*M*L*K outputs, the first 2*M*L*K the sampling offsets in level
    pixels in [M, L, K, 2] order, the last M*L*K the attention logits in
    [M, L*K] order; then locations = ref + offsets / (W_l, H_l) and the
    softmax over each (b, q, m)'s L*K logits.  query [B, Q, C].
    Returns (sampling_locations [B,Q,M,L,K,2], attention_weights [B,Q,M,L,K])."""
    y = linear(query, weight, bias)
    B, Q = y.shape[0], y.shape[1]
    P = M * L * K
    assert y.shape[2] == 3 * P
    off = np.ascontiguousarray(y[:, :, :2 * P]).reshape(B, Q, M, L, K, 2)
    logits = np.ascontiguousarray(y[:, :, 2 * P:]).reshape(B, Q, M, L * K)
    return sampling_locations(spatial_shapes, reference_points, off), softmax(logits, L, K)


def query_head_backward(spatial_shapes, attention_weights, grad_loc, grad_attn):
    """Gradient of the query head's linear outputs [B, Q, 3*M*L*K] (offsets
    then logits, the weight's row order) and of the reference points
    [B, Q, 2], from the core's grad_sampling_locations and
    grad_attention_weights: the chain rule of query_head's location and
    softmax steps (fused_chain)."""
    goff, gref, glog = fused_chain(spatial_shapes, attention_weights, grad_loc, grad_attn, True)
    B, Q = goff.shape[0], goff.shape[1]
    return np.concatenate([goff.reshape(B, Q, -1), glog.reshape(B, Q, -1)], axis=2), gref
