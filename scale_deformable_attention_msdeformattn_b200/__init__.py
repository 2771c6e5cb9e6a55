"""B200-native (sm_100a) multi-scale deformable attention core.

The operator runs in libmsda.so (hand-written CUDA kernels behind the C ABI of
include/msda.h); this package is its Python binding.  PyTorch only provides
device memory and the current stream, and, in the optional MSDeformAttn layer,
the linear projections around the operator.
"""
from .module import MSDeformAttn  # noqa: F401
from .binding import (  # noqa: F401
    MsdaError,
    MSDeformAttnFunction,
    MSDeformAttnFusedFunction,
    backward,
    backward_noalloc,
    DCNv3CoreFunction,
    dcn_backward,
    dcn_forward,
    dcnv3_core,
    device_status,
    forward,
    fused_backward,
    fused_forward,
    linear,
    ms_deform_attn,
    quantize_value_e4m3,
    quantize_value_s8,
    query_head,
    query_head_backward,
    sort_queries,
    version,
    zero_grads,
)

__version__ = "0.1.0"
