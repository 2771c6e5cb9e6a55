"""Python binding of the C-ABI: torch tensors in, libmsda.so calls, tensors out.

Only argument marshalling happens here (shape and dtype checks, output
allocation through PyTorch, pointer and stream hand-off).  Every step of the
operator runs in the CUDA kernels of libmsda.so; there is no CPU or PyTorch
fallback, and a missing library raises.

Layouts follow the operator's conventional argument list (cf-1.com/news/4799680
§5.3, x-humanoid.csdn.net MSDA explainer §3):
  value               [B, S, M, D]        float32 or bfloat16
  spatial_shapes      [L, 2]  int64 (H, W)
  level_start_index   [L]     int64
  sampling_locations  [B, Q, M, L, K, 2]  float32, normalized (x, y)
  attention_weights   [B, Q, M, L, K]     float32
  reference_points    [B, Q, 2]           float32 (fused variant)
  sampling_offsets    [B, Q, M, L, K, 2]  float32, level pixels (fused variant)
  attention_logits    [B, Q, M, L*K] or [B, Q, M, L, K] float32 (fused variant)
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _lib


class MsdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _lib.load()
        msg = lib.msda_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


def _check(status: int, where: str):
    if status != _lib.MSDA_OK:
        raise MsdaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr()) if t.numel() > 0 else None


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


_DTYPES = {torch.float32: _lib.MSDA_F32, torch.bfloat16: _lib.MSDA_BF16, torch.int8: _lib.MSDA_S8,
           torch.float8_e4m3fn: _lib.MSDA_E4M3}
# one-byte value storage: codes times a (batch, head) scale (value_scale)
_SCALED = (torch.int8, torch.float8_e4m3fn)


def _row_dtype(value: torch.Tensor):
    """dtype of output / grad_output: value's, bfloat16 for one-byte value."""
    return torch.bfloat16 if value.dtype in _SCALED else value.dtype


def _problem(value: torch.Tensor, Q: int, L: int, K: int, flags: int = 0,
             query_order: Optional[torch.Tensor] = None,
             value_scale: Optional[torch.Tensor] = None) -> _lib.Problem:
    if value.dim() != 4:
        raise ValueError("value must be [B, S, M, D]")
    if value.dtype not in _DTYPES:
        raise TypeError("value must be float32, bfloat16, int8 or float8_e4m3fn (with value_scale)")
    B, S, M, D = value.shape
    prob = _lib.Problem(B, S, Q, M, D, L, K, _DTYPES[value.dtype], flags)
    if value.dtype in _SCALED:
        if value_scale is None:
            raise ValueError("one-byte value needs value_scale [B, M] "
                             "(see quantize_value_s8, quantize_value_e4m3)")
        _need(value_scale, "value_scale", torch.float32, (B, M), value.device)
        prob.value_scale = _ptr(value_scale)
    if query_order is not None:
        if query_order.numel() != B * Q:
            raise ValueError(f"query_order must hold B*Q = {B * Q} entries")
        _need(query_order, "query_order", torch.int32, None, value.device)
        prob.query_order = _ptr(query_order)
    return prob


def _geometry(value, spatial_shapes, level_start_index):
    _need(spatial_shapes, "spatial_shapes", torch.int64, device=value.device)
    if spatial_shapes.dim() != 2 or spatial_shapes.shape[1] != 2:
        raise ValueError("spatial_shapes must be [L, 2]")
    L = spatial_shapes.shape[0]
    _need(level_start_index, "level_start_index", torch.int64, (L,), device=value.device)
    return L


def forward(value: torch.Tensor, spatial_shapes: torch.Tensor, level_start_index: torch.Tensor,
            sampling_locations: torch.Tensor, attention_weights: torch.Tensor,
            out: Optional[torch.Tensor] = None,
            query_order: Optional[torch.Tensor] = None,
            value_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """msda_forward: returns out [B, Q, M, D] in value's dtype (bfloat16 for
    one-byte value, which needs value_scale [B, M]).  query_order: optional int32
    [B*Q] processing order (see sort_queries)."""
    _need(value, "value", None)
    L = _geometry(value, spatial_shapes, level_start_index)
    B, S, M, D = value.shape
    if sampling_locations.dim() != 6:
        raise ValueError("sampling_locations must be [B, Q, M, L, K, 2]")
    Q, K = sampling_locations.shape[1], sampling_locations.shape[4]
    _need(sampling_locations, "sampling_locations", torch.float32, (B, Q, M, L, K, 2), value.device)
    _need(attention_weights, "attention_weights", torch.float32, (B, Q, M, L, K), value.device)
    if out is None:
        out = torch.empty((B, Q, M, D), dtype=_row_dtype(value), device=value.device)
    _need(out, "out", _row_dtype(value), (B, Q, M, D), value.device)
    prob = _problem(value, Q, L, K, 0, query_order, value_scale)
    st = _lib.load().msda_forward(ctypes.byref(prob), _ptr(value), _ptr(spatial_shapes),
                                  _ptr(level_start_index), _ptr(sampling_locations),
                                  _ptr(attention_weights), _ptr(out), _stream())
    _check(st, "msda_forward")
    return out


def backward(value, spatial_shapes, level_start_index, sampling_locations, attention_weights,
             grad_output, grad_value_dtype=torch.float32,
             grad_value: Optional[torch.Tensor] = None,
             grad_sampling_locations: Optional[torch.Tensor] = None,
             grad_attention_weights: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None,
             accumulate: bool = False,
             query_order: Optional[torch.Tensor] = None,
             value_scale: Optional[torch.Tensor] = None,
             merge_reductions: bool = False) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """msda_backward: (grad_value, grad_sampling_locations, grad_attention_weights).

    accumulate=True adds into the given float32 grad_value instead of
    overwriting it (MSDA_ACCUMULATE_GRADS); merge_reductions=True merges the
    grad_value contributions of each tile per corner row before reducing them
    (MSDA_MERGE_REDUCTIONS, a performance option)."""
    _need(value, "value", None)
    L = _geometry(value, spatial_shapes, level_start_index)
    B, S, M, D = value.shape
    Q, K = sampling_locations.shape[1], sampling_locations.shape[4]
    dev = value.device
    _need(sampling_locations, "sampling_locations", torch.float32, (B, Q, M, L, K, 2), dev)
    _need(attention_weights, "attention_weights", torch.float32, (B, Q, M, L, K), dev)
    _need(grad_output, "grad_output", _row_dtype(value), (B, Q, M, D), dev)
    flags = _lib.MSDA_GRAD_VALUE_BF16 if grad_value_dtype == torch.bfloat16 else 0
    if grad_value_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("grad_value_dtype must be float32 or bfloat16")
    if accumulate:
        if grad_value is None:
            raise ValueError("accumulate=True needs the grad_value buffer to add into")
        flags |= _lib.MSDA_ACCUMULATE_GRADS
    if merge_reductions:
        flags |= _lib.MSDA_MERGE_REDUCTIONS
    if grad_value is None:
        grad_value = torch.empty((B, S, M, D), dtype=grad_value_dtype, device=dev)
    if grad_sampling_locations is None:
        grad_sampling_locations = torch.empty((B, Q, M, L, K, 2), dtype=torch.float32, device=dev)
    if grad_attention_weights is None:
        grad_attention_weights = torch.empty((B, Q, M, L, K), dtype=torch.float32, device=dev)
    _need(grad_value, "grad_value", grad_value_dtype, (B, S, M, D), dev)
    prob = _problem(value, Q, L, K, flags, query_order, value_scale)
    lib = _lib.load()
    ws_bytes = ctypes.c_size_t(0)
    _check(lib.msda_backward_workspace_size(ctypes.byref(prob), ctypes.byref(ws_bytes)),
           "msda_backward_workspace_size")
    if ws_bytes.value and workspace is None:
        workspace = torch.empty(ws_bytes.value, dtype=torch.uint8, device=dev)
    st = lib.msda_backward(ctypes.byref(prob), _ptr(value), _ptr(spatial_shapes),
                           _ptr(level_start_index), _ptr(sampling_locations),
                           _ptr(attention_weights), _ptr(grad_output), _ptr(grad_value),
                           _ptr(grad_sampling_locations), _ptr(grad_attention_weights),
                           _ptr(workspace), workspace.numel() if workspace is not None else 0,
                           _stream())
    _check(st, "msda_backward")
    return grad_value, grad_sampling_locations, grad_attention_weights


def _logits(attention_logits, B, Q, M, L, K, dev):
    if attention_logits.dim() == 5:
        attention_logits = attention_logits.reshape(B, Q, M, L * K)
    return _need(attention_logits, "attention_logits", torch.float32, (B, Q, M, L * K), dev)


def fused_forward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                  attention_logits, return_attention_weights: bool = False,
                  out: Optional[torch.Tensor] = None,
                  query_order: Optional[torch.Tensor] = None,
                  value_scale: Optional[torch.Tensor] = None):
    """msda_fused_forward: out [B, Q, M, D] (and the softmax weights if asked)."""
    _need(value, "value", None)
    L = _geometry(value, spatial_shapes, level_start_index)
    B, S, M, D = value.shape
    if sampling_offsets.dim() != 6:
        raise ValueError("sampling_offsets must be [B, Q, M, L, K, 2]")
    Q, K = sampling_offsets.shape[1], sampling_offsets.shape[4]
    dev = value.device
    _need(reference_points, "reference_points", torch.float32, (B, Q, 2), dev)
    _need(sampling_offsets, "sampling_offsets", torch.float32, (B, Q, M, L, K, 2), dev)
    attention_logits = _logits(attention_logits, B, Q, M, L, K, dev)
    if out is None:
        out = torch.empty((B, Q, M, D), dtype=_row_dtype(value), device=dev)
    _need(out, "out", _row_dtype(value), (B, Q, M, D), dev)
    attn = torch.empty((B, Q, M, L, K), dtype=torch.float32, device=dev) if return_attention_weights else None
    prob = _problem(value, Q, L, K, 0, query_order, value_scale)
    st = _lib.load().msda_fused_forward(ctypes.byref(prob), _ptr(value), _ptr(spatial_shapes),
                                        _ptr(level_start_index), _ptr(reference_points),
                                        _ptr(sampling_offsets), _ptr(attention_logits), _ptr(out),
                                        _ptr(attn), _stream())
    _check(st, "msda_fused_forward")
    return (out, attn) if return_attention_weights else out


def fused_backward(value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                   attention_logits, grad_output, grad_value_dtype=torch.float32,
                   want_grad_reference_points: bool = True,
                   grad_value: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   accumulate: bool = False,
                   grad_reference_points: Optional[torch.Tensor] = None,
                   grad_sampling_offsets: Optional[torch.Tensor] = None,
                   grad_attention_logits: Optional[torch.Tensor] = None,
                   query_order: Optional[torch.Tensor] = None,
                   value_scale: Optional[torch.Tensor] = None,
                   merge_reductions: bool = False):
    """msda_fused_backward: (grad_value, grad_reference_points or None,
    grad_sampling_offsets, grad_attention_logits [B, Q, M, L*K]).

    accumulate=True adds into the given float32 grad_value (and
    grad_reference_points) instead of overwriting them; merge_reductions=True
    merges each tile's grad_value contributions per corner row first
    (MSDA_MERGE_REDUCTIONS, a performance option)."""
    _need(value, "value", None)
    L = _geometry(value, spatial_shapes, level_start_index)
    B, S, M, D = value.shape
    Q, K = sampling_offsets.shape[1], sampling_offsets.shape[4]
    dev = value.device
    _need(reference_points, "reference_points", torch.float32, (B, Q, 2), dev)
    _need(sampling_offsets, "sampling_offsets", torch.float32, (B, Q, M, L, K, 2), dev)
    attention_logits = _logits(attention_logits, B, Q, M, L, K, dev)
    _need(grad_output, "grad_output", _row_dtype(value), (B, Q, M, D), dev)
    if grad_value_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("grad_value_dtype must be float32 or bfloat16")
    flags = _lib.MSDA_GRAD_VALUE_BF16 if grad_value_dtype == torch.bfloat16 else 0
    if accumulate:
        if grad_value is None or (want_grad_reference_points and grad_reference_points is None):
            raise ValueError("accumulate=True needs the buffers to add into")
        flags |= _lib.MSDA_ACCUMULATE_GRADS
    if merge_reductions:
        flags |= _lib.MSDA_MERGE_REDUCTIONS
    if grad_value is None:
        grad_value = torch.empty((B, S, M, D), dtype=grad_value_dtype, device=dev)
    _need(grad_value, "grad_value", grad_value_dtype, (B, S, M, D), dev)
    gref = None
    if want_grad_reference_points:
        gref = grad_reference_points if grad_reference_points is not None else \
            torch.empty((B, Q, 2), dtype=torch.float32, device=dev)
        _need(gref, "grad_reference_points", torch.float32, (B, Q, 2), dev)
    goff = grad_sampling_offsets if grad_sampling_offsets is not None else \
        torch.empty((B, Q, M, L, K, 2), dtype=torch.float32, device=dev)
    _need(goff, "grad_sampling_offsets", torch.float32, (B, Q, M, L, K, 2), dev)
    glog = grad_attention_logits if grad_attention_logits is not None else \
        torch.empty((B, Q, M, L * K), dtype=torch.float32, device=dev)
    _need(glog, "grad_attention_logits", torch.float32, (B, Q, M, L * K), dev)
    prob = _problem(value, Q, L, K, flags, query_order, value_scale)
    lib = _lib.load()
    ws_bytes = ctypes.c_size_t(0)
    _check(lib.msda_backward_workspace_size(ctypes.byref(prob), ctypes.byref(ws_bytes)),
           "msda_backward_workspace_size")
    if ws_bytes.value and workspace is None:
        workspace = torch.empty(ws_bytes.value, dtype=torch.uint8, device=dev)
    st = lib.msda_fused_backward(ctypes.byref(prob), _ptr(value), _ptr(spatial_shapes),
                                 _ptr(level_start_index), _ptr(reference_points),
                                 _ptr(sampling_offsets), _ptr(attention_logits), _ptr(grad_output),
                                 _ptr(grad_value), _ptr(gref), _ptr(goff), _ptr(glog),
                                 _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                 _stream())
    _check(st, "msda_fused_backward")
    return grad_value, gref, goff, glog


def backward_noalloc(value, spatial_shapes, level_start_index, sampling_locations,
                     attention_weights, grad_output, grad_value: Optional[torch.Tensor] = None,
                     grad_sampling_locations: Optional[torch.Tensor] = None,
                     grad_attention_weights: Optional[torch.Tensor] = None):
    """msda_backward_noalloc: backward with grad_value written as bf16, using
    the library's own float32 scratch buffer instead of a workspace (for
    callers that cannot allocate device memory when they run the backward).
    Pass preallocated outputs to keep this call itself allocation-free."""
    _need(value, "value", None)
    L = _geometry(value, spatial_shapes, level_start_index)
    B, S, M, D = value.shape
    Q, K = sampling_locations.shape[1], sampling_locations.shape[4]
    dev = value.device
    _need(sampling_locations, "sampling_locations", torch.float32, (B, Q, M, L, K, 2), dev)
    _need(attention_weights, "attention_weights", torch.float32, (B, Q, M, L, K), dev)
    _need(grad_output, "grad_output", value.dtype, (B, Q, M, D), dev)
    if grad_value is None:
        grad_value = torch.empty((B, S, M, D), dtype=torch.bfloat16, device=dev)
    if grad_sampling_locations is None:
        grad_sampling_locations = torch.empty((B, Q, M, L, K, 2), dtype=torch.float32, device=dev)
    if grad_attention_weights is None:
        grad_attention_weights = torch.empty((B, Q, M, L, K), dtype=torch.float32, device=dev)
    _need(grad_value, "grad_value", torch.bfloat16, (B, S, M, D), dev)
    prob = _problem(value, Q, L, K, _lib.MSDA_GRAD_VALUE_BF16)
    st = _lib.load().msda_backward_noalloc(ctypes.byref(prob), _ptr(value), _ptr(spatial_shapes),
                                           _ptr(level_start_index), _ptr(sampling_locations),
                                           _ptr(attention_weights), _ptr(grad_output),
                                           _ptr(grad_value), _ptr(grad_sampling_locations),
                                           _ptr(grad_attention_weights), _stream())
    _check(st, "msda_backward_noalloc")
    return grad_value, grad_sampling_locations, grad_attention_weights


def quantize_value_s8(value: torch.Tensor, value_s8: Optional[torch.Tensor] = None,
                      value_scale: Optional[torch.Tensor] = None):
    """msda_quantize_value_s8: (int8 value [B, S, M, D], float32 scale [B, M])
    from a float32 or bfloat16 value, one symmetric absmax scale per
    (batch, head); pass both to the other calls (value_scale=...)."""
    _need(value, "value", None)
    if value.dim() != 4 or value.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("value must be a float32 or bfloat16 [B, S, M, D] tensor")
    B, S, M, D = value.shape
    if value_s8 is None:
        value_s8 = torch.empty((B, S, M, D), dtype=torch.int8, device=value.device)
    if value_scale is None:
        value_scale = torch.empty((B, M), dtype=torch.float32, device=value.device)
    _need(value_s8, "value_s8", torch.int8, (B, S, M, D), value.device)
    _need(value_scale, "value_scale", torch.float32, (B, M), value.device)
    prob = _lib.Problem(B, S, 1, M, D, 1, 1, _DTYPES[value.dtype], 0)
    st = _lib.load().msda_quantize_value_s8(ctypes.byref(prob), _ptr(value), _ptr(value_s8),
                                            _ptr(value_scale), _stream())
    _check(st, "msda_quantize_value_s8")
    return value_s8, value_scale


def quantize_value_e4m3(value: torch.Tensor, value_e4m3: Optional[torch.Tensor] = None,
                        value_scale: Optional[torch.Tensor] = None):
    """msda_quantize_value_e4m3: (float8_e4m3fn value [B, S, M, D], float32
    scale [B, M]) from a float32 or bfloat16 value, one absmax scale per
    (batch, head), amax / 448; pass both to the other calls
    (value_scale=...)."""
    _need(value, "value", None)
    if value.dim() != 4 or value.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("value must be a float32 or bfloat16 [B, S, M, D] tensor")
    B, S, M, D = value.shape
    if value_e4m3 is None:
        value_e4m3 = torch.empty((B, S, M, D), dtype=torch.float8_e4m3fn, device=value.device)
    if value_scale is None:
        value_scale = torch.empty((B, M), dtype=torch.float32, device=value.device)
    _need(value_e4m3, "value_e4m3", torch.float8_e4m3fn, (B, S, M, D), value.device)
    _need(value_scale, "value_scale", torch.float32, (B, M), value.device)
    prob = _lib.Problem(B, S, 1, M, D, 1, 1, _DTYPES[value.dtype], 0)
    st = _lib.load().msda_quantize_value_e4m3(ctypes.byref(prob), _ptr(value), _ptr(value_e4m3),
                                              _ptr(value_scale), _stream())
    _check(st, "msda_quantize_value_e4m3")
    return value_e4m3, value_scale


def _pair(v):
    return (int(v), int(v)) if isinstance(v, int) else (int(v[0]), int(v[1]))


def _dcn_problem(input: torch.Tensor, kernel, stride, pad, dilation, flags=0, value_scale=None):
    if input.dim() != 5:
        raise ValueError("input must be [N, H, W, G, C]")
    if input.dtype not in _DTYPES:
        raise TypeError("input must be float32, bfloat16, int8 or float8_e4m3fn (with value_scale)")
    N, H, W, G, C = input.shape
    (kh, kw), (sh, sw), (ph, pw), (dh, dw) = _pair(kernel), _pair(stride), _pair(pad), _pair(dilation)
    prob = _lib.DcnProblem(N, H, W, G, C, kh, kw, sh, sw, ph, pw, dh, dw, _DTYPES[input.dtype], flags)
    if input.dtype in _SCALED:
        if value_scale is None:
            raise ValueError("one-byte input needs value_scale [N, G] "
                             "(see quantize_value_s8, quantize_value_e4m3)")
        _need(value_scale, "value_scale", torch.float32, (N, G), input.device)
        prob.value_scale = _ptr(value_scale)
    ho, wo = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(_lib.load().msda_dcn_output_size(ctypes.byref(prob), ctypes.byref(ho), ctypes.byref(wo)),
           "msda_dcn_output_size")
    return prob, ho.value, wo.value


def dcn_forward(input: torch.Tensor, offset: torch.Tensor, mask: torch.Tensor, kernel=3, stride=1,
                pad=1, dilation=1, out: Optional[torch.Tensor] = None,
                value_scale: Optional[torch.Tensor] = None) -> torch.Tensor:
    """msda_dcn_forward (DCNv3 core): input [N,H,W,G,C], offset [N,Ho,Wo,G,K,2]
    (dx, dy) pixels, mask [N,Ho,Wo,G,K] (used as given) -> [N,Ho,Wo,G,C]."""
    _need(input, "input", None)
    prob, Ho, Wo = _dcn_problem(input, kernel, stride, pad, dilation, 0, value_scale)
    N, H, W, G, C = input.shape
    K = prob.kernel_h * prob.kernel_w
    dev = input.device
    _need(offset, "offset", torch.float32, (N, Ho, Wo, G, K, 2), dev)
    _need(mask, "mask", torch.float32, (N, Ho, Wo, G, K), dev)
    if out is None:
        out = torch.empty((N, Ho, Wo, G, C), dtype=_row_dtype(input), device=dev)
    _need(out, "out", _row_dtype(input), (N, Ho, Wo, G, C), dev)
    st = _lib.load().msda_dcn_forward(ctypes.byref(prob), _ptr(input), _ptr(offset), _ptr(mask),
                                      _ptr(out), _stream())
    _check(st, "msda_dcn_forward")
    return out


def dcn_backward(input, offset, mask, grad_output, kernel=3, stride=1, pad=1, dilation=1,
                 grad_input_dtype=torch.float32, grad_input: Optional[torch.Tensor] = None,
                 accumulate: bool = False, value_scale: Optional[torch.Tensor] = None,
                 grad_offset: Optional[torch.Tensor] = None,
                 grad_mask: Optional[torch.Tensor] = None,
                 merge_reductions: bool = False):
    """msda_dcn_backward: (grad_input, grad_offset, grad_mask);
    merge_reductions=True merges each tile's contributions per input row
    before reducing them (MSDA_MERGE_REDUCTIONS)."""
    _need(input, "input", None)
    if grad_input_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("grad_input_dtype must be float32 or bfloat16")
    flags = _lib.MSDA_GRAD_VALUE_BF16 if grad_input_dtype == torch.bfloat16 else 0
    if accumulate:
        if grad_input is None:
            raise ValueError("accumulate=True needs the grad_input buffer to add into")
        flags |= _lib.MSDA_ACCUMULATE_GRADS
    if merge_reductions:
        flags |= _lib.MSDA_MERGE_REDUCTIONS
    prob, Ho, Wo = _dcn_problem(input, kernel, stride, pad, dilation, flags, value_scale)
    N, H, W, G, C = input.shape
    K = prob.kernel_h * prob.kernel_w
    dev = input.device
    _need(offset, "offset", torch.float32, (N, Ho, Wo, G, K, 2), dev)
    _need(mask, "mask", torch.float32, (N, Ho, Wo, G, K), dev)
    _need(grad_output, "grad_output", _row_dtype(input), (N, Ho, Wo, G, C), dev)
    if grad_input is None:
        grad_input = torch.empty((N, H, W, G, C), dtype=grad_input_dtype, device=dev)
    _need(grad_input, "grad_input", grad_input_dtype, (N, H, W, G, C), dev)
    goff = grad_offset if grad_offset is not None else torch.empty_like(offset)
    gmask = grad_mask if grad_mask is not None else torch.empty_like(mask)
    _need(goff, "grad_offset", torch.float32, tuple(offset.shape), dev)
    _need(gmask, "grad_mask", torch.float32, tuple(mask.shape), dev)
    lib = _lib.load()
    ws_bytes = ctypes.c_size_t(0)
    _check(lib.msda_dcn_backward_workspace_size(ctypes.byref(prob), ctypes.byref(ws_bytes)),
           "msda_dcn_backward_workspace_size")
    workspace = torch.empty(ws_bytes.value, dtype=torch.uint8, device=dev) if ws_bytes.value else None
    st = lib.msda_dcn_backward(ctypes.byref(prob), _ptr(input), _ptr(offset), _ptr(mask),
                               _ptr(grad_output), _ptr(grad_input), _ptr(goff), _ptr(gmask),
                               _ptr(workspace), ws_bytes.value, _stream())
    _check(st, "msda_dcn_backward")
    return grad_input, goff, gmask


# ------------------------------------------------ dense layers (tcgen05) --

def linear(x: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None, out_dtype=torch.float32) -> torch.Tensor:
    """msda_linear: x [..., K] bf16 @ weight[N, K]^T (+ bias [N] float32) on the
    tensor cores, float32 accumulation; returns [..., N] in out_dtype (float32
    or bfloat16).  K must be a multiple of 8."""
    if x.dtype != torch.bfloat16 or weight.dtype != torch.bfloat16:
        raise TypeError("x and weight must be bfloat16")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out_dtype must be float32 or bfloat16")
    N, K = weight.shape
    if x.shape[-1] != K:
        raise ValueError(f"x has {x.shape[-1]} features, weight expects {K}")
    dev = x.device
    _need(x, "x", torch.bfloat16, None, dev)
    _need(weight, "weight", torch.bfloat16, (N, K), dev)
    if bias is not None:
        _need(bias, "bias", torch.float32, (N,), dev)
    rows = x.numel() // K if K else 0
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=out_dtype, device=dev)
    _need(out, "out", out_dtype, tuple(x.shape[:-1]) + (N,), dev)
    st = _lib.load().msda_linear(rows, K, N, _ptr(x), _ptr(weight), _ptr(bias), _ptr(out),
                                 _DTYPES[out_dtype], _stream())
    _check(st, "msda_linear")
    return out


def _head_problem(B, Q, M, L, K):
    return _lib.Problem(B, 0, Q, M, 0, L, K, _lib.MSDA_F32, 0)


def query_head(query: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor],
               reference_points: torch.Tensor, spatial_shapes: torch.Tensor, num_heads: int,
               num_points: int, sampling_locations: Optional[torch.Tensor] = None,
               attention_weights: Optional[torch.Tensor] = None):
    """msda_query_head: the offset / logit head (weight [3*M*L*K, C] bf16, rows
    in [offsets (M, L, K, 2) | logits (M, L*K)] order) fused with the location
    step and the softmax.  query [B, Q, C] bf16.  Returns
    (sampling_locations [B,Q,M,L,K,2], attention_weights [B,Q,M,L,K])."""
    if query.dtype != torch.bfloat16 or weight.dtype != torch.bfloat16:
        raise TypeError("query and weight must be bfloat16")
    B, Q, C = query.shape
    L = spatial_shapes.shape[0]
    M, K = num_heads, num_points
    P = M * L * K
    dev = query.device
    _need(query, "query", torch.bfloat16, (B, Q, C), dev)
    _need(weight, "weight", torch.bfloat16, (3 * P, C), dev)
    if bias is not None:
        _need(bias, "bias", torch.float32, (3 * P,), dev)
    _need(reference_points, "reference_points", torch.float32, (B, Q, 2), dev)
    _need(spatial_shapes, "spatial_shapes", torch.int64, (L, 2), dev)
    loc = sampling_locations if sampling_locations is not None else \
        torch.empty((B, Q, M, L, K, 2), dtype=torch.float32, device=dev)
    attn = attention_weights if attention_weights is not None else \
        torch.empty((B, Q, M, L, K), dtype=torch.float32, device=dev)
    _need(loc, "sampling_locations", torch.float32, (B, Q, M, L, K, 2), dev)
    _need(attn, "attention_weights", torch.float32, (B, Q, M, L, K), dev)
    prob = _head_problem(B, Q, M, L, K)
    st = _lib.load().msda_query_head(ctypes.byref(prob), C, _ptr(query), _ptr(weight), _ptr(bias),
                                     _ptr(reference_points), _ptr(spatial_shapes), _ptr(loc),
                                     _ptr(attn), _stream())
    _check(st, "msda_query_head")
    return loc, attn


def query_head_backward(attention_weights: torch.Tensor, grad_sampling_locations: torch.Tensor,
                        grad_attention_weights: torch.Tensor, spatial_shapes: torch.Tensor,
                        want_grad_reference_points: bool = False):
    """msda_query_head_backward: (grad_head [B, Q, 3*M*L*K] float32, the
    gradient of the head's linear outputs; grad_reference_points [B, Q, 2] or
    None)."""
    B, Q, M, L, K = attention_weights.shape
    P = M * L * K
    dev = attention_weights.device
    _need(attention_weights, "attention_weights", torch.float32, (B, Q, M, L, K), dev)
    _need(grad_sampling_locations, "grad_sampling_locations", torch.float32, (B, Q, M, L, K, 2), dev)
    _need(grad_attention_weights, "grad_attention_weights", torch.float32, (B, Q, M, L, K), dev)
    _need(spatial_shapes, "spatial_shapes", torch.int64, (L, 2), dev)
    gh = torch.empty((B, Q, 3 * P), dtype=torch.float32, device=dev)
    gref = torch.empty((B, Q, 2), dtype=torch.float32, device=dev) if want_grad_reference_points else None
    prob = _head_problem(B, Q, M, L, K)
    st = _lib.load().msda_query_head_backward(ctypes.byref(prob), _ptr(attention_weights),
                                              _ptr(grad_sampling_locations), _ptr(grad_attention_weights),
                                              _ptr(spatial_shapes), _ptr(gh), _ptr(gref), _stream())
    _check(st, "msda_query_head_backward")
    return gh, gref


def sort_queries(points: torch.Tensor, query_order: Optional[torch.Tensor] = None) -> torch.Tensor:
    """msda_sort_queries: int32 [B*Q] order of the queries by batch, then by
    the Morton code of the 64 x 64 cell of [0,1]^2 holding points[b, q]
    (float32 [B, Q, 2], e.g. the reference points).  Pass the result as
    query_order to the other calls."""
    _need(points, "points", torch.float32)
    if points.dim() != 3 or points.shape[2] != 2:
        raise ValueError("points must be [B, Q, 2]")
    B, Q = points.shape[0], points.shape[1]
    dev = points.device
    prob = _lib.Problem(B, 1, Q, 1, 8, 1, 1, _lib.MSDA_F32, 0)
    if query_order is None:
        query_order = torch.empty(B * Q, dtype=torch.int32, device=dev)
    _need(query_order, "query_order", torch.int32, (B * Q,), dev)
    st = _lib.load().msda_sort_queries(ctypes.byref(prob), _ptr(points), _ptr(query_order), _stream())
    _check(st, "msda_sort_queries")
    return query_order


def zero_grads(grad_value: torch.Tensor, grad_reference_points: Optional[torch.Tensor] = None,
               num_queries: int = 0, num_levels: int = 1, num_points: int = 1):
    """msda_zero_grads: zeroes float32 grad_value [B, S, M, D] (and
    grad_reference_points [B, Q, 2]) in a library kernel."""
    _need(grad_value, "grad_value", torch.float32)
    B, S, M, D = grad_value.shape
    Q = grad_reference_points.shape[1] if grad_reference_points is not None else num_queries
    if grad_reference_points is not None:
        _need(grad_reference_points, "grad_reference_points", torch.float32, (B, Q, 2), grad_value.device)
    prob = _lib.Problem(B, S, Q, M, D, num_levels, num_points, _lib.MSDA_F32, 0)
    st = _lib.load().msda_zero_grads(ctypes.byref(prob), _ptr(grad_value), _ptr(grad_reference_points),
                                     _stream())
    _check(st, "msda_zero_grads")


def device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronizes the stream and returns (and clears) the kernels' status word."""
    s = ctypes.c_void_p((stream or torch.cuda.current_stream()).cuda_stream)
    code = ctypes.c_int32(0)
    _check(_lib.load().msda_get_device_status(s, ctypes.byref(code)), "msda_get_device_status")
    return code.value


def version() -> str:
    return _lib.load().msda_version().decode()


class MSDeformAttnFunction(torch.autograd.Function):
    """Autograd wrapper over msda_forward / msda_backward (grad_value in the
    value's dtype).  Same argument order as the operator's usual autograd
    function; a trailing im2col_step is accepted and ignored (the kernels
    have no column buffer to chunk), so existing call sites need no change."""

    @staticmethod
    def forward(ctx, value, spatial_shapes, level_start_index, sampling_locations, attention_weights,
                im2col_step=None):
        ctx.save_for_backward(value, spatial_shapes, level_start_index, sampling_locations,
                              attention_weights)
        return forward(value, spatial_shapes, level_start_index, sampling_locations,
                       attention_weights)

    @staticmethod
    def backward(ctx, grad_output):
        value, shapes, starts, loc, attn = ctx.saved_tensors
        gv, gl, ga = backward(value, shapes, starts, loc, attn, grad_output.contiguous(),
                              grad_value_dtype=value.dtype)
        return gv, None, None, gl, ga, None


class MSDeformAttnFusedFunction(torch.autograd.Function):
    """Autograd wrapper over msda_fused_forward / msda_fused_backward."""

    @staticmethod
    def forward(ctx, value, spatial_shapes, level_start_index, reference_points, sampling_offsets,
                attention_logits):
        ctx.save_for_backward(value, spatial_shapes, level_start_index, reference_points,
                              sampling_offsets, attention_logits)
        return fused_forward(value, spatial_shapes, level_start_index, reference_points,
                             sampling_offsets, attention_logits)

    @staticmethod
    def backward(ctx, grad_output):
        value, shapes, starts, ref, off, logits = ctx.saved_tensors
        gv, gref, goff, glog = fused_backward(value, shapes, starts, ref, off, logits,
                                              grad_output.contiguous(), grad_value_dtype=value.dtype)
        return gv, None, None, gref, goff, glog.reshape(logits.shape)


def ms_deform_attn(value, spatial_shapes, level_start_index, sampling_locations, attention_weights,
                   im2col_step=None):
    """Differentiable core operator; output [B, Q, M*D] like the module's
    reshape before output_proj (im2col_step accepted and ignored)."""
    out = MSDeformAttnFunction.apply(value, spatial_shapes, level_start_index, sampling_locations,
                                     attention_weights, im2col_step)
    return out.flatten(2)


class DCNv3CoreFunction(torch.autograd.Function):
    """Autograd wrapper over msda_dcn_forward / msda_dcn_backward (float32 or
    bfloat16 input; grad_input in the input's dtype)."""

    @staticmethod
    def forward(ctx, input, offset, mask, kernel=3, stride=1, pad=1, dilation=1):
        ctx.save_for_backward(input, offset, mask)
        ctx.geo = dict(kernel=kernel, stride=stride, pad=pad, dilation=dilation)
        return dcn_forward(input, offset, mask, **ctx.geo)

    @staticmethod
    def backward(ctx, grad_output):
        input, offset, mask = ctx.saved_tensors
        gx, goff, gm = dcn_backward(input, offset, mask, grad_output.contiguous(),
                                    grad_input_dtype=input.dtype, **ctx.geo)
        return gx, goff, gm, None, None, None, None


def dcnv3_core(input, offset, mask, kernel=3, stride=1, pad=1, dilation=1):
    """Differentiable DCNv3 core: [N, H, W, G, C] -> [N, Ho, Wo, G*C] (the
    layout the group projection w_g consumes)."""
    return DCNv3CoreFunction.apply(input, offset, mask, kernel, stride, pad, dilation).flatten(3)
