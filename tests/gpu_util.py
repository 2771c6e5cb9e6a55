"""Helpers shared by the GPU tests: upload seeded inputs, run the oracle,
compare.  Two error metrics per output tensor, both asserted:

  normwise    max_i |gpu_i - ref_i| / max_i |ref_i|
  elementwise max_i |gpu_i - ref_i| / max(|ref_i|, 1e-3 * max_j |ref_j|)

The normwise bound is the stated precision target (1e-5 for float32 value,
2e-2 for bf16 value with float32 accumulation).  The elementwise metric keeps
a large error on a small element from hiding under the largest one; its
floor of 1e-3 * max|ref| stops elements that cancel to (near) zero from
dividing by nothing.  Its bounds: float32 outputs 1e-3 (float32 accumulation
over at most a few hundred terms is ~1e-6 of the terms' magnitude, which a
cancelled element at the floor sees magnified up to 1000x); outputs stored
as bf16 2e-2 (round to nearest even is within 2^-9 relative of the float32
sum, plus that sum's own error)."""
import numpy as np
import torch

import oracle
from scale_deformable_attention_msdeformattn_b200 import workloads as wl

# tolerances of the two precision regimes (float32 value; bf16 value with
# float32 accumulation), for forward and backward outputs alike
TOL = {"f32": 1e-5, "bf16": 2e-2}
# elementwise bounds (floor 1e-3 * max|ref|): float32 outputs, bf16 outputs
ELEM_TOL = {"f32": 1e-3, "bf16": 2e-2}
ELEM_FLOOR = 1e-3


def value_tensor(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype in ("bf16", "s8", "e4m3"):  # one-byte workloads carry the bf16 source
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


def elem_err(gpu, ref, floor: float = ELEM_FLOOR) -> float:
    g = host(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if g.size == 0:
        return 0.0
    if not np.isfinite(g).all():
        return float("inf")
    scale = np.abs(r).max()
    if scale == 0.0:
        return float(np.abs(g - r).max())
    return float((np.abs(g - r) / np.maximum(np.abs(r), floor * scale)).max())


# (what, normwise error, elementwise error) of every assert_close call, for
# the run's summary table (tests/conftest.py)
RECORDS = []


def assert_close(gpu, ref, tol, what, elem_tol=None, floor=ELEM_FLOOR):
    """Asserts the normwise error <= tol and the elementwise error <= elem_tol
    (default: ELEM_TOL for bf16 tensors, else for float32) with the given
    floor; prints both."""
    e = rel_err(gpu, ref)
    if elem_tol is None:
        is_bf16 = isinstance(gpu, torch.Tensor) and gpu.dtype == torch.bfloat16
        elem_tol = ELEM_TOL["bf16" if is_bf16 else "f32"]
    ee = elem_err(gpu, ref, floor)
    print(f"  {what}: normwise {e:.2e} elementwise {ee:.2e}")
    RECORDS.append((what, e, ee))
    assert e <= tol, f"{what}: max relative error {e:.3e} > {tol:.1e}"
    assert ee <= elem_tol, f"{what}: elementwise relative error {ee:.3e} > {elem_tol:.1e}"
    return e


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bf16 (nearest even), widened back to float64."""
    return wl.bf16_bits_to_f64(wl.to_bf16_bits(x))


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
