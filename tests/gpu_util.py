"""Helpers shared by the GPU tests: upload seeded inputs, run the oracle,
compare.  The comparison metric is the normwise maximum relative error
max_i |gpu_i - ref_i| / max_i |ref_i| of each output tensor."""
import numpy as np
import torch

import oracle
from scale_deformable_attention_msdeformattn_b200 import workloads as wl

# tolerances of the two precision regimes (float32 value; bf16 value with
# float32 accumulation), for forward and backward outputs alike
TOL = {"f32": 1e-5, "bf16": 2e-2}


def value_tensor(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype in ("bf16", "s8"):  # s8 workloads carry the bf16 source
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(arr).to(device)


def upload(x: wl.Inputs, device="cuda"):
    w = x.workload
    t = dict(
        value=value_tensor(x.value, w.dtype, device),
        spatial_shapes=torch.from_numpy(x.spatial_shapes).to(device),
        level_start_index=torch.from_numpy(x.level_start_index).to(device),
        reference_points=torch.from_numpy(x.reference_points).to(device),
        sampling_offsets=torch.from_numpy(x.sampling_offsets).to(device),
        attention_logits=torch.from_numpy(x.attention_logits).to(device),
        grad_output=value_tensor(x.grad_output, w.dtype, device),
    )
    if x.sampling_locations.size:
        t["sampling_locations"] = torch.from_numpy(x.sampling_locations).to(device)
        t["attention_weights"] = torch.from_numpy(x.attention_weights).to(device)
    return t


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(gpu, ref) -> float:
    g = host(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return 0.0
    if not np.isfinite(g).all():
        return float("inf")
    scale = np.abs(r).max()
    err = np.abs(g - r).max()
    if scale == 0.0:
        return float(err)
    return float(err / scale)


def assert_close(gpu, ref, tol, what):
    e = rel_err(gpu, ref)
    assert e <= tol, f"{what}: max relative error {e:.3e} > {tol:.1e}"
    return e


def oracle_nonfused(x: wl.Inputs):
    v, g = x.value_f64(), x.grad_output_f64()
    out = oracle.forward(v, x.spatial_shapes, x.level_start_index, x.sampling_locations,
                         x.attention_weights)
    gv, gl, ga = oracle.backward(v, x.spatial_shapes, x.level_start_index, x.sampling_locations,
                                 x.attention_weights, g)
    return out, gv, gl, ga


def oracle_fused(x: wl.Inputs):
    v, g = x.value_f64(), x.grad_output_f64()
    out, a, loc = oracle.fused_forward(v, x.spatial_shapes, x.level_start_index, x.reference_points,
                                       x.sampling_offsets, x.attention_logits)
    gv, gref, goff, glog = oracle.fused_backward(v, x.spatial_shapes, x.level_start_index,
                                                 x.reference_points, x.sampling_offsets,
                                                 x.attention_logits, g)
    return out, a, gv, gref, goff, glog
