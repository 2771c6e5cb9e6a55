"""Query-ordered processing: msda_sort_queries and the optional query_order
of msda_problem (the query-sorting step of the operator's data-locality
notes, x-humanoid.csdn.net MSDA explainer §4).  The order changes which rows a
CTA handles together, never what a row computes, so every output is compared
with the oracle exactly as in the natural order, and the non-fused forward is
compared bit for bit with the natural order."""
import numpy as np
import pytest
import torch

import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, oracle_fused, oracle_nonfused, upload

pytestmark = pytest.mark.gpu


def _morton_cell_key(points: np.ndarray) -> np.ndarray:
    """(batch, Morton code of the 64 x 64 cell) of every point, bit by bit."""
    B, Q, _ = points.shape
    p = points.astype(np.float32)
    with np.errstate(invalid="ignore"):
        cell = np.floor(np.clip(np.nan_to_num(p * np.float32(64), nan=0.0), 0, 63)).astype(np.int64)
    cx, cy = cell[..., 0], cell[..., 1]
    code = np.zeros_like(cx)
    for bit in range(6):
        code |= ((cx >> bit) & 1) << (2 * bit)
        code |= ((cy >> bit) & 1) << (2 * bit + 1)
    return (np.arange(B)[:, None] * 4096 + code).reshape(-1)


def _check_sorted_permutation(order: torch.Tensor, points: np.ndarray):
    o = order.cpu().numpy().astype(np.int64)
    n = points.shape[0] * points.shape[1]
    assert o.shape == (n,)
    assert np.array_equal(np.sort(o), np.arange(n)), "not a permutation"
    keys = _morton_cell_key(points)[o]
    assert np.all(np.diff(keys) >= 0), "keys not ascending along the order"


def test_sort_queries_orders_by_batch_and_cell():
    g = np.random.default_rng(7)
    B, Q = 3, 5000
    pts = g.uniform(-0.2, 1.2, size=(B, Q, 2)).astype(np.float32)
    pts[0, :7] = [[0.0, 0.0], [1.0, 1.0], [np.nan, 0.5], [0.5, np.inf], [-np.inf, 2.0],
                  [63.5 / 64, 0.25], [1 / 64, 1 / 64]]
    t = torch.from_numpy(pts).cuda()
    order = msda.sort_queries(t)
    assert msda.device_status() == 0
    _check_sorted_permutation(order, pts)
    # a second call into a caller buffer gives an order of the same keys
    out = torch.full((B * Q,), -1, dtype=torch.int32, device="cuda")
    msda.sort_queries(t, query_order=out)
    _check_sorted_permutation(out, pts)


def test_sort_queries_large_batch_of_queries():
    """More queries than one pass of the sort's CTA covers (several passes,
    ragged tail), batch-major keys."""
    g = np.random.default_rng(8)
    B, Q = 2, 3 * 8192 + 77
    pts = g.uniform(0.0, 1.0, size=(B, Q, 2)).astype(np.float32)
    pts[1, ::5] = 0.5  # a crowded cell
    order = msda.sort_queries(torch.from_numpy(pts).cuda())
    _check_sorted_permutation(order, pts)


def _nonfused(t, order=None):
    out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                       t["sampling_locations"], t["attention_weights"], query_order=order)
    grads = msda.backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                          t["sampling_locations"], t["attention_weights"], t["grad_output"],
                          query_order=order)
    return (out,) + grads


def _fused(t, order=None):
    out, attn = msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                                   t["reference_points"], t["sampling_offsets"],
                                   t["attention_logits"], return_attention_weights=True,
                                   query_order=order)
    grads = msda.fused_backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                                t["reference_points"], t["sampling_offsets"], t["attention_logits"],
                                t["grad_output"], query_order=order)
    return (out, attn) + grads


def _compare(w, x, t, order):
    tol = TOL[w.dtype]
    got = _nonfused(t, order)
    assert msda.device_status() == 0
    nat = _nonfused(t)
    assert torch.equal(got[0], nat[0]), "forward output depends on the order"
    assert torch.equal(got[2], nat[2]) and torch.equal(got[3], nat[3]), \
        "per-sample gradients depend on the order"
    ref = oracle_nonfused(x)
    for g, r, what in zip(got, ref, ("out", "grad_value", "grad_loc", "grad_attn")):
        assert_close(g, r, tol, f"{w.name} ordered {what}")
    got = _fused(t, order)
    assert msda.device_status() == 0
    r_out, r_a, r_gv, r_gref, r_goff, r_glog = oracle_fused(x)
    for g, r, what in zip(got, (r_out, r_a, r_gv, r_gref, r_goff, r_glog),
                          ("out", "attn", "grad_value", "grad_ref", "grad_off", "grad_logits")):
        assert_close(g, r, tol, f"{w.name} ordered fused {what}")


@pytest.mark.parametrize("name", ["detr_decoder_bf16", "detr_encoder_f32"])
def test_sorted_order_full_size(name):
    """Full-size workloads processed in the order msda_sort_queries gives for
    their reference points, the configuration the bench times with --sorted."""
    w = wl.WORKLOADS[name]
    x = wl.generate(w)
    t = upload(x)
    order = msda.sort_queries(t["reference_points"])
    _check_sorted_permutation(order, x.reference_points)
    _compare(w, x, t, order)


@pytest.mark.parametrize("spec", [
    ("perm_ragged_f32", 3, [(11, 13), (6, 7), (3, 4)], None, 8, 32, 4, "f32", "pixel_centre", 2.0),
    ("perm_bf16_d64", 2, [(13, 17), (7, 9)], 29, 4, 64, 2, "bf16", "uniform", 3.0),
    ("perm_k32", 1, [(20, 30), (10, 15), (5, 8), (3, 4)], 45, 2, 32, 32, "f32", "uniform", 3.0),
])
def test_random_permutation(spec):
    """Any permutation is a valid order (not only sorted ones)."""
    name, B, levels, Q, M, D, K, dtype, ref, sigma = spec
    w = wl.custom(name, B, levels, Q, M, D, K, dtype, ref, sigma, 1.0, index=500 + len(name))
    x = wl.generate(w)
    t = upload(x)
    g = torch.Generator().manual_seed(11)
    order = torch.randperm(w.B * w.num_queries, generator=g).to(torch.int32).cuda()
    _compare(w, x, t, order)


def test_out_of_range_order_entry_is_reported():
    """An entry outside 0 .. B*Q-1 is caught by the kernels (no fault): it is
    replaced by query 0 and the status word says MSDA_ERR_DEVICE_CHECK."""
    w = wl.WORKLOADS["tiny_f32"]
    x = wl.generate(w)
    t = upload(x)
    n = w.B * w.num_queries
    assert msda.device_status() == 0
    order = torch.arange(n, dtype=torch.int32, device="cuda")
    order[3] = n
    order[5] = -7
    out = msda.forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                       t["sampling_locations"], t["attention_weights"], query_order=order)
    assert msda.device_status() == 4
    assert torch.isfinite(out.flatten(0, 1)[0]).all()
    msda.fused_backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                        t["reference_points"], t["sampling_offsets"], t["attention_logits"],
                        t["grad_output"], query_order=order)
    assert msda.device_status() == 4
    assert msda.device_status() == 0


def test_order_with_no_queries_is_ignored():
    w = wl.custom("empty_order", 1, [(4, 5), (2, 3)], 1, 2, 16, 2, "f32", index=530)
    t = upload(wl.generate(w))
    v = t["value"]
    loc = torch.zeros((1, 0, 2, 2, 2, 2), device="cuda")
    a = torch.zeros((1, 0, 2, 2, 2), device="cuda")
    order = torch.empty(0, dtype=torch.int32, device="cuda")
    out = msda.forward(v, t["spatial_shapes"], t["level_start_index"], loc, a, query_order=order)
    assert out.shape == (1, 0, 2, 16)
    assert msda.sort_queries(torch.zeros((1, 0, 2), device="cuda")).numel() == 0
    assert msda.device_status() == 0
