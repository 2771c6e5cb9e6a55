"""The attention calls inside a CUDA graph: the fused forward, the zero-fill
on a second stream and the accumulating fused backward, captured once after
a warm-up call and replayed; the replays reproduce the launched results (the
forward bit for bit, the gradients within the float32 tolerance, as their
reduction order varies)."""
import pytest
import torch

import scale_deformable_attention_msdeformattn_b200 as msda
from scale_deformable_attention_msdeformattn_b200 import workloads as wl
from tests.gpu_util import TOL, assert_close, upload

pytestmark = pytest.mark.gpu


def test_fused_step_replays_from_a_cuda_graph():
    w = wl.custom("graph", 2, [(20, 30), (10, 15), (5, 8)], 97, 8, 32, 4, "f32", index=800)
    t = upload(wl.generate(w))
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    dev = t["value"].device
    out = torch.empty((B, Q, M, D), device=dev)
    gv = torch.empty((B, S, M, D), device=dev)
    gref = torch.empty((B, Q, 2), device=dev)
    goff = torch.empty((B, Q, M, L, K, 2), device=dev)
    glog = torch.empty((B, Q, M, L * K), device=dev)
    side = torch.cuda.Stream()

    def step():
        cur = torch.cuda.current_stream()
        fork, join = torch.cuda.Event(), torch.cuda.Event()
        fork.record(cur)
        side.wait_event(fork)
        with torch.cuda.stream(side):
            msda.zero_grads(gv, gref)
            join.record(side)
        msda.fused_forward(t["value"], t["spatial_shapes"], t["level_start_index"],
                           t["reference_points"], t["sampling_offsets"], t["attention_logits"], out=out)
        cur.wait_event(join)
        msda.fused_backward(t["value"], t["spatial_shapes"], t["level_start_index"],
                            t["reference_points"], t["sampling_offsets"], t["attention_logits"],
                            t["grad_output"], accumulate=True, grad_value=gv, grad_reference_points=gref,
                            grad_sampling_offsets=goff, grad_attention_logits=glog)

    step()
    torch.cuda.synchronize()
    ref = [x.clone() for x in (out, gv, gref, goff, glog)]
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            step()
    torch.cuda.current_stream().wait_stream(cap)
    for x in (out, gv, gref, goff, glog):
        x.fill_(float("nan"))
    for _ in range(2):  # the zero-fill inside the graph resets the accumulators
        g.replay()
    torch.cuda.synchronize()
    assert msda.device_status() == 0
    assert torch.equal(out, ref[0])
    for got, want, what in zip((gv, gref, goff, glog), ref[1:],
                               ("grad_value", "grad_ref", "grad_off", "grad_logits")):
        assert_close(got, want.double().cpu().numpy(), TOL["f32"], f"graph replay {what}")
    del g
