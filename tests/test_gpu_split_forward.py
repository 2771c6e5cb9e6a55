"""The forward with rows split over lane groups (taken when a problem's rows,
one lane group each, would not fill one resident wave of the GPU: the
decoder's 300 queries per image) and the unsplit forward, on both sides of
that threshold, against the oracle.

Small problems everywhere else in the suite take the split kernel; these
cases put the head dims the split serves (float32 D = 8, 16, 32; bf16 D = 8
... 64 with at most 16 samples per row) just above the threshold too, so
that their unsplit kernels meet the oracle as well.  The threshold depends
on the SM count, read from the device."""
import pytest
import torch

import oracle
import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, upload

pytestmark = pytest.mark.gpu

LEVELS = [(23, 31), (12, 16), (6, 8), (3, 4)]
VB = 16  # bytes per lane vector of the forward


def _rows_per_warp(D: int, dtype: str) -> int:
    lanes = max(1, min(32, D * {"f32": 4, "bf16": 2}[dtype] // VB))
    return 32 // lanes


def _threshold_rows(D: int, dtype: str) -> int:
    """Rows at which the launcher stops splitting: one resident wave of the
    unsplit kernel (8 warps per CTA; 4 CTAs per SM for float32, 3 for bf16
    rows of at most 16 samples)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ctas = 4 if dtype == "f32" else 3
    return sms * 8 * ctas * _rows_per_warp(D, dtype)


@pytest.mark.parametrize("side", ["split", "unsplit"])
@pytest.mark.parametrize("D,dtype", [(8, "f32"), (16, "f32"), (32, "f32"), (8, "bf16"),
                                     (16, "bf16"), (32, "bf16"), (64, "bf16")])
def test_forward_across_split_threshold(D, dtype, side):
    M, K = 4, 4
    rows = _threshold_rows(D, dtype)
    # a ragged count of queries below, or at and above, the threshold
    Q = (rows // M) - 37 if side == "split" else (rows // M) + 5
    w = wl.custom(f"split_{side}_{dtype}_{D}", 1, LEVELS, Q, M, D, K, dtype, "uniform", 3.0, 1.0,
                  index=700 + D + (1 if dtype == "bf16" else 0))
    x = wl.generate(w, with_nonfused=True)
    t = upload(x)
    geo = (t["spatial_shapes"], t["level_start_index"])
    out = msda.forward(t["value"], *geo, t["sampling_locations"], t["attention_weights"])
    fout = msda.fused_forward(t["value"], *geo, t["reference_points"], t["sampling_offsets"],
                              t["attention_logits"])
    assert msda.device_status() == 0
    v = x.value_f64()
    want = oracle.forward(v, x.spatial_shapes, x.level_start_index, x.sampling_locations,
                          x.attention_weights)
    fwant, _, _ = oracle.fused_forward(v, x.spatial_shapes, x.level_start_index, x.reference_points,
                                       x.sampling_offsets, x.attention_logits)
    tol = TOL[dtype]
    assert_close(out, want, tol, f"{w.name} out")
    assert_close(fout, fwant, tol, f"{w.name} fused out")
