"""The step bench.py times, in its own launch configuration, against the fp64
oracle at full size: the fused forward on the current stream, the zero-fill
of the gradient accumulators on a second stream beside it, and the fused
backward accumulating into them once both are done; three steps back to
back with an L2 flush in between, as the bench runs them, then every output
of the last step compared element by element with the oracle."""
import pytest
import torch

import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, oracle_fused, upload

pytestmark = pytest.mark.gpu

L2_FLUSH_FLOATS = (256 << 20) // 4  # a write larger than the 126 MB L2


def _bench_step(t, o, side):
    cur = torch.cuda.current_stream()
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    fork.record(cur)
    msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"], t["reference_points"],
                       t["sampling_offsets"], t["attention_logits"], out=o["out"])
    side.wait_event(fork)
    with torch.cuda.stream(side):
        msda.zero_grads(o["grad_value"], o["grad_reference_points"])
        join.record(side)
    cur.wait_event(join)
    msda.fused_backward(t["value"], t["spatial_shapes"], t["level_start_index"], t["reference_points"],
                        t["sampling_offsets"], t["attention_logits"], t["grad_output"], accumulate=True,
                        grad_value=o["grad_value"], grad_reference_points=o["grad_reference_points"],
                        grad_sampling_offsets=o["grad_sampling_offsets"],
                        grad_attention_logits=o["grad_attention_logits"])


@pytest.mark.parametrize("name", ["detr_encoder_f32", "detr_decoder_bf16"])
def test_bench_step_matches_oracle(name):
    w = wl.WORKLOADS[name]
    x = wl.generate(w, with_nonfused=False)
    t = upload(x)
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    dev = t["value"].device
    o = {"out": torch.empty((B, Q, M, D), dtype=t["value"].dtype, device=dev),
         "grad_value": torch.full((B, S, M, D), float("nan"), device=dev),
         "grad_reference_points": torch.full((B, Q, 2), float("nan"), device=dev),
         "grad_sampling_offsets": torch.empty((B, Q, M, L, K, 2), device=dev),
         "grad_attention_logits": torch.empty((B, Q, M, L * K), device=dev)}
    side = torch.cuda.Stream()
    flush = torch.empty(L2_FLUSH_FLOATS, device=dev)
    for i in range(3):
        flush.fill_(float(i))
        _bench_step(t, o, side)
    torch.cuda.synchronize()
    assert msda.device_status() == 0
    r_out, _, r_gv, r_gref, r_goff, r_glog = oracle_fused(x)
    tol = TOL[w.dtype]
    assert_close(o["out"], r_out, tol, f"{name} bench step out")
    assert_close(o["grad_value"], r_gv, tol, f"{name} bench step grad_value")
    assert_close(o["grad_reference_points"], r_gref, tol, f"{name} bench step grad_reference_points")
    assert_close(o["grad_sampling_offsets"], r_goff, tol, f"{name} bench step grad_sampling_offsets")
    assert_close(o["grad_attention_logits"], r_glog, tol, f"{name} bench step grad_attention_logits")
