#!/usr/bin/env python
"""Throughput of the multi-scale deformable attention core on B200.

One step = one pass of the whole hot path over one batch of the workload:
msda_fused_forward (location step, softmax over L*K, bilinear gather,
weighted sum), msda_zero_grads (float32 gradient accumulators) and
msda_fused_backward (gathers again, gradients of the sample, grad_value
scatter, chain rule to offsets, reference points and logits).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Prints one JSON line on rank 0.  `value` is G sampled points per second over
the fwd+bwd step (samples = B*Q*M*L*K per step, all ranks), with inputs
resident in HBM and L2 flushed between steps; each kernel is timed with CUDA
events on the stream it is launched on.  Multi-GPU runs (torchrun, one process
per GPU) give every rank its own batch of the workload (weak scaling; there is
no data-path collective).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from scale_deformable_attention_msdeformattn_b200 import workloads as wl  # noqa: E402

METRIC = "G sampled points/s and fwd+bwd ms at DETR-encoder shape; % of B200 HBM roofline"
UNIT = "G samples/s"
L2_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, one launch) of
# the kernels as last captured with ncu, keyed by kernel; each entry records the
# hash of the CUDA sources it was taken from and is reported only while those
# sources are unchanged.  Filled from the summaries under profiles/.
NCU_TRAFFIC = {
    # DRAM read + write per launch (the mean of the launches captured), from
    # the counter captures listed in the profiles/ summaries
    ("fused_backward", "detr_encoder_f32"): {"bytes": 126197632, "csrc": "9ceaf8a65da5ceee"},
    ("fused_forward", "detr_encoder_f32"): {"bytes": 59481600, "csrc": "9ceaf8a65da5ceee"},
    ("fused_backward", "detr_decoder_bf16"): {"bytes": 132292352, "csrc": "9ceaf8a65da5ceee"},
    ("fused_forward", "detr_decoder_bf16"): {"bytes": 51024640, "csrc": "9ceaf8a65da5ceee"},
    ("fused_backward", "stress_1080p_k8_bf16"): {"bytes": 914386688, "csrc": "9ceaf8a65da5ceee"},
    ("fused_forward", "stress_1080p_k8_bf16"): {"bytes": 381361664, "csrc": "9ceaf8a65da5ceee"},
    ("dcn_backward", "dcnv3_stage1_f32"): {"bytes": 140071168, "csrc": "9ceaf8a65da5ceee"},
    ("dcn_forward", "dcnv3_stage1_f32"): {"bytes": 73025024, "csrc": "9ceaf8a65da5ceee"},
}


def _code_only(text: str) -> str:
    """C++ source without its comments and blank lines (a comment edit keeps
    the hash)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def csrc_hash() -> str:
    """Hash of the code the operator kernels are compiled and launched from:
    every file of csrc/ except the dense-layer GEMM header (which none of
    them includes), comments left out."""
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "scale_deformable_attention_msdeformattn_b200",
                                           "csrc", "*"))):
        if os.path.basename(p) == "msda_gemm.cuh":
            continue
        with open(p, encoding="utf-8") as f:
            h.update(os.path.basename(p).encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="detr_encoder_f32",
                    choices=sorted(wl.WORKLOADS) + sorted(wl.DCN_WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="host-core seconds spent timing the oracle for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-nonfused", action="store_true")
    ap.add_argument("--layer", action="store_true",
                    help="time the whole MSDeformAttn layer (tensor-core projections and fused "
                         "query head around the core), forward + backward, at the workload's "
                         "shape with C = M*D, beside torch linear layers around the fused core")
    ap.add_argument("--merge-reductions", action="store_true",
                    help="backward merges each tile's grad_value contributions per corner "
                         "row before reducing them (MSDA_MERGE_REDUCTIONS)")
    ap.add_argument("--zero", choices=("overlap", "serial"), default="overlap",
                    help="where the zero-fill of the gradient accumulators runs: on a second "
                         "stream beside the forward (default), or after it on the launch stream")
    ap.add_argument("--sorted", action="store_true",
                    help="order the queries by the Morton cell of their reference point "
                         "(msda_sort_queries, inside the timed step) and process them in that order")
    ap.add_argument("--headline", choices=("graph", "launched"), default="graph",
                    help="what `value` times: the step replayed from a CUDA graph captured once "
                         "(default), or the step's calls launched one by one from the host; the "
                         "other is reported beside it")
    ap.add_argument("--out", default=None, help="also append the JSON line to this file")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


# ---------------------------------------------------------------- bytes ----

def algorithmic_bytes(w: wl.Workload) -> dict:
    """Each tensor of a launch touched once (inputs read, outputs written)."""
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    e = {"f32": 4, "bf16": 2, "s8": 1, "e4m3": 1}[w.dtype]       # value element
    er = {"f32": 4, "bf16": 2, "s8": 2, "e4m3": 2}[w.dtype]      # output / grad_output element
    value = B * S * M * D * e
    rowd = B * Q * M * D * er
    samples = B * Q * M * L * K
    loc = samples * 2 * 4
    attn = samples * 4
    ref = B * Q * 2 * 4
    gvalue = B * S * M * D * 4
    fwd = value + loc + attn + rowd
    bwd = rowd + value + loc + attn + gvalue + loc + attn
    fused_fwd = value + loc + attn + ref + rowd             # offsets, logits, ref -> out
    fused_bwd = rowd + value + loc + attn + ref + gvalue + loc + attn + ref
    # INT8 storage: the bf16 source read once, the codes written once
    quantize = B * S * M * D * 3 if w.dtype in ("s8", "e4m3") else 0
    return {"forward": fwd, "backward": bwd, "fused_forward": fused_fwd,
            "fused_backward": fused_bwd, "zero_grads": gvalue + ref, "quantize": quantize}


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    """Polls NVML for the SM clock and the clock-event reasons of one GPU."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_device: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[torch_device]) if vis and vis.split(",")[0].isdigit() else torch_device
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self._reasons_fn(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"error": "NVML unavailable: " + getattr(self, "err", "")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(mhz), "reasons": reasons, "samples": len(mhz)}


# ------------------------------------------------------------- our arm -----

def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_workload(base: wl.Workload, rank: int) -> wl.Workload:
    """Weak scaling: every rank processes its own batch of the workload (its
    own seed), with no exchange between ranks."""
    return base if rank == 0 else wl.dataclasses.replace(base, index=base.index + 1000 * rank)


def _other_timing(headline: str, graph_ok: bool, steps: int, launched, graph) -> dict:
    """The JSON entry of the step timing that is not the headline: value,
    ms per step and percentiles of (value, total ms, per-step ms)."""
    if not graph_ok:
        return {"graph": {"unavailable": "CUDA graph capture failed; the launched steps are the headline"}}
    key, (v, total, ms) = ("launched", launched) if headline == "graph" else ("graph", graph)
    return {key: {"value": round(v, 4), "unit": UNIT, "ms_per_step": round(total / steps, 5),
                  "step_ms_p10_p50_p90": [round(float(np.percentile(ms, p)), 5) for p in (10, 50, 90)]}}


def _all_ranks(ok: bool, world: int, device=None) -> bool:
    """Whether ok holds on every rank (a MIN all-reduce when world > 1)."""
    if world == 1:
        return ok
    import torch
    import torch.distributed as dist
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def aggregate_over_ranks(total_ms: float, samples_per_rank_step: int, steps: int, world: int,
                         device=None):
    """Max over ranks of the timed duration (ms) and the whole-job throughput
    in G samples/s.  Collective over the default process group when world > 1
    (any backend: NCCL on GPUs, gloo in the CPU tests)."""
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([total_ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * samples_per_rank_step * steps / (total_ms * 1e-3) / 1e9
    return total_ms, value


def _to_device(x: wl.Inputs, dev):
    import torch

    def val(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    t = {
        "value": val(x.value),
        "spatial_shapes": torch.from_numpy(x.spatial_shapes).to(dev),
        "level_start_index": torch.from_numpy(x.level_start_index).to(dev),
        "reference_points": torch.from_numpy(x.reference_points).to(dev),
        "sampling_offsets": torch.from_numpy(x.sampling_offsets).to(dev),
        "attention_logits": torch.from_numpy(x.attention_logits).to(dev),
        "grad_output": val(x.grad_output),
    }
    if x.sampling_locations.size:
        t["sampling_locations"] = torch.from_numpy(x.sampling_locations).to(dev)
        t["attention_weights"] = torch.from_numpy(x.attention_weights).to(dev)
    return t


def _pinned(x: wl.Inputs):
    """Host copies of one step's inputs in pinned memory (for the e2e leg)."""
    import torch

    def pin(a):
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(a)
        return t.pin_memory()

    return {k: pin(v) for k, v in {
        "value": x.value, "spatial_shapes": x.spatial_shapes,
        "level_start_index": x.level_start_index, "reference_points": x.reference_points,
        "sampling_offsets": x.sampling_offsets, "attention_logits": x.attention_logits,
        "grad_output": x.grad_output}.items()}


def run_ours(args):
    import torch
    import torch.distributed as dist
    import scale_deformable_attention_msdeformattn_b200 as msda

    world, rank, local = _dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = rank_workload(wl.WORKLOADS[args.workload], rank)
    want_nonfused = not args.no_nonfused and world == 1
    x = wl.generate(w, with_nonfused=want_nonfused)
    t = _to_device(x, dev)
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    def make_outputs():
        return {"out": torch.empty((B, Q, M, D), dtype=t["value"].dtype, device=dev),
                "grad_value": torch.empty((B, S, M, D), dtype=torch.float32, device=dev),
                "grad_reference_points": torch.empty((B, Q, 2), dtype=torch.float32, device=dev),
                "grad_sampling_offsets": torch.empty((B, Q, M, L, K, 2), dtype=torch.float32, device=dev),
                "grad_attention_logits": torch.empty((B, Q, M, L * K), dtype=torch.float32, device=dev)}

    outputs = make_outputs()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    side = torch.cuda.Stream(device=dev)
    order = torch.empty(B * Q, dtype=torch.int32, device=dev) if args.sorted else None
    # one-byte value storage: the step's value arrives as bf16 and is stored
    # as INT8 or FP8 codes with a (batch, head) scale
    int8 = w.dtype in ("s8", "e4m3")
    qdtype, quantize = ((torch.int8, lambda v, q, sc: msda.quantize_value_s8(v, value_s8=q, value_scale=sc))
                        if w.dtype == "s8" else
                        (torch.float8_e4m3fn,
                         lambda v, q, sc: msda.quantize_value_e4m3(v, value_e4m3=q, value_scale=sc)))
    qv = torch.empty((B, S, M, D), dtype=qdtype, device=dev) if int8 else None
    qs = torch.empty((B, M), dtype=torch.float32, device=dev) if int8 else None

    nbytes = algorithmic_bytes(w)
    overlap = args.zero == "overlap"

    def step(ev, tin=None, o=None):
        # the zero-fill of the gradient accumulators does not depend on the
        # forward: it runs on a second stream beside it and the backward waits
        # for both (--zero serial puts it after the forward instead: decoder
        # step 137 against 129 us, but the forward's own time without HBM
        # shared with the zero-fill's 182 MB)
        tin = tin or t
        o = o or outputs
        stream = torch.cuda.current_stream()  # the capture stream under graph capture
        ev[0].record(stream)
        if order is not None:
            msda.sort_queries(tin["reference_points"], query_order=order)
        if int8:  # the step's value arrives as bf16 and is stored in one byte
            quantize(tin["value"], qv, qs)
        value = qv if int8 else tin["value"]
        ev[6].record(stream)
        msda.fused_forward(value, tin["spatial_shapes"], tin["level_start_index"],
                           tin["reference_points"], tin["sampling_offsets"],
                           tin["attention_logits"], out=o["out"], query_order=order, value_scale=qs)
        if overlap:  # enqueued after the forward, whose CTAs take the SMs first
            side.wait_event(ev[6])
            with torch.cuda.stream(side):
                ev[4].record(side)
                msda.zero_grads(o["grad_value"], o["grad_reference_points"])
                ev[5].record(side)
        ev[1].record(stream)
        if overlap:
            stream.wait_event(ev[5])
        else:
            ev[4].record(stream)
            msda.zero_grads(o["grad_value"], o["grad_reference_points"])
            ev[5].record(stream)
        ev[2].record(stream)
        msda.fused_backward(value, tin["spatial_shapes"], tin["level_start_index"],
                            tin["reference_points"], tin["sampling_offsets"],
                            tin["attention_logits"], tin["grad_output"], accumulate=True,
                            grad_value=o["grad_value"], grad_reference_points=o["grad_reference_points"],
                            grad_sampling_offsets=o["grad_sampling_offsets"],
                            grad_attention_logits=o["grad_attention_logits"],
                            query_order=order, value_scale=qs,
                            merge_reductions=args.merge_reductions)
        ev[3].record(stream)
        return o

    def events(n):
        return [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(n)]

    warm = events(args.warmup)
    for i in range(args.warmup):
        flush.fill_(float(i))
        step(warm[i])
    torch.cuda.synchronize()
    if msda.device_status() != 0:
        raise SystemExit("kernels reported inconsistent geometry")

    # K launched steps: the per-kernel times (events between the calls)
    evs = events(args.steps)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    wall0 = time.perf_counter()
    for i in range(args.steps):
        flush.fill_(float(i))  # L2 flush, outside the timed events
        step(evs[i])
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier()

    # K replays of the same step from a CUDA graph: the step without the
    # host's launch gaps
    graphms = _graph_steps(step, 7, flush, args.steps, barrier, lambda ok: _all_ranks(ok, world, dev))
    clocks.stop()
    if msda.device_status() != 0:
        raise SystemExit("kernels reported inconsistent geometry")

    fwd = [e[6].elapsed_time(e[1]) for e in evs]
    pre = [e[0].elapsed_time(e[6]) for e in evs]
    zero = [e[4].elapsed_time(e[5]) for e in evs]
    bwd = [e[2].elapsed_time(e[3]) for e in evs]
    stepms = [e[0].elapsed_time(e[3]) for e in evs]
    samples_step = w.samples
    l_total_ms, l_value = aggregate_over_ranks(float(sum(stepms)), samples_step, args.steps, world, dev)
    graph_ok = graphms is not None
    if not graph_ok:  # no graph: the launched steps are the headline
        args.headline, graphms = "launched", stepms
    g_total_ms, g_value = aggregate_over_ranks(float(sum(graphms)), samples_step, args.steps, world, dev)
    if args.headline == "graph":
        total_ms, value, headms = g_total_ms, g_value, graphms
    else:
        total_ms, value, headms = l_total_ms, l_value, stepms
    ms_per_step = total_ms / args.steps

    result = None
    if rank == 0:
        peaks = _peaks()
        fwd_ms, bwd_ms, zero_ms = statistics.mean(fwd), statistics.mean(bwd), statistics.mean(zero)
        dom = "fused_backward" if bwd_ms >= fwd_ms else "fused_forward"
        dom_ms = bwd_ms if dom == "fused_backward" else fwd_ms
        achieved = nbytes[dom] / (dom_ms * 1e-3) / 1e9
        tr = NCU_TRAFFIC.get((dom, w.name))
        traffic = tr["bytes"] if tr and tr.get("csrc") == csrc_hash() else None
        step_bytes = nbytes["fused_forward"] + nbytes["fused_backward"] + nbytes["quantize"]
        result = {
            "metric": METRIC,
            "value": round(value, 4),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"f32": "f32", "bf16": "bf16 value / f32 accumulate",
                      "s8": "int8 value (per batch-head scale) / bf16 rows / f32 accumulate",
                      "e4m3": "fp8 e4m3 value (per batch-head scale) / bf16 rows / f32 accumulate"}[w.dtype],
            "data": "synthetic: seeded SplitMix64 + Box-Muller draws of the workload's shapes "
                    "and distributions (no dataset)",
            "config": {
                "workload": w.name, "B": w.B, "levels_HW": [list(l) for l in w.levels],
                "Q": Q, "M": M, "D": D, "L": L, "K": K,
                "offset_sigma_px": w.offset_sigma, "logit_sigma": w.logit_sigma,
                "samples_per_step_per_gpu": samples_step,
                "step": ("msda_sort_queries -> " if args.sorted else "")
                + (f"msda_quantize_value_{w.dtype} -> " if int8 else "")
                + ("msda_fused_forward || msda_zero_grads (second stream) -> msda_fused_backward"
                   if overlap else "msda_fused_forward -> msda_zero_grads -> msda_fused_backward"),
                "query_order": "Morton cell of the reference point" if args.sorted else "natural",
                "l2": "flushed between steps (256 MiB write outside the timed events)",
                "timing": ("the step replayed from a CUDA graph captured once (both streams), events "
                           "around each replay" if args.headline == "graph" else
                           "the step's calls launched one by one, events around each step"),
                "parallelism": f"dp{world} (independent batch per GPU)",
            },
            "fwd_ms": round(fwd_ms, 5),
            "zero_ms": round(zero_ms, 5),  # under the forward, or after it (config.step)
            # before the forward: the query sort (--sorted) and the INT8 quantisation
            "pre_ms": round(statistics.mean(pre), 5) if (args.sorted or int8) else None,

            "bwd_ms": round(bwd_ms, 5),
            "fwd_gsamples_per_s": round(samples_step / (fwd_ms * 1e-3) / 1e9, 4),
            "step_ms_p10_p50_p90": [round(float(np.percentile(headms, p)), 5) for p in (10, 50, 90)],
            # the other way of timing the same step (config.timing names the headline's)
            **_other_timing(args.headline, graph_ok, args.steps, (l_value, l_total_ms, stepms),
                            (g_value, g_total_ms, graphms)),
            "hbm_frac_step": round(step_bytes / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "roofline": {
                "kernel": dom,
                "bound": "hbm",
                "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"],
                "peak_source": peaks["source"],
                "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "bytes_per_launch": nbytes[dom],
                "traffic": traffic,
            },
            "gpu_launches": (3 + (1 if args.sorted else 0) + (3 if int8 else 0)) * args.steps,
            "host_wall_s": round(wall, 3),
            "clocks": clocks.summary(),
        }
        if want_nonfused:
            if int8:
                quantize(t["value"], qv, qs)
            result["nonfused"] = _time_nonfused(msda, t, w, nbytes, flush, min(args.steps, 50),
                                                qv if int8 else t["value"], qs)
        if world == 1:
            # the fused backward with the other grad_value reduction path
            result["bwd_other_reductions"] = _time_bwd(
                msda, t, o=outputs, flush=flush, n=min(args.steps, 50),
                value=qv if int8 else t["value"], value_scale=qs, order=order,
                merge=not args.merge_reductions)
            result["config"]["grad_value_reductions"] = (
                "merged per tile of consecutive queries of one head"
                if args.merge_reductions and not args.sorted
                else "direct (one vector reduction per corner contribution)")
            result["fwd_alone"] = _time_fwd(msda, t, outputs, flush, min(args.steps, 50),
                                            qv if int8 else t["value"], qs, order, nbytes, peaks)
            result["warm_l2"] = _time_warm(w, step, min(args.steps, 50))
        stats = _input_stats(w, x)
        if "value_bytes_touched" in stats:
            # the value tensor counted by the sectors the gathers touch instead of whole
            touched = step_bytes - 2 * (stats["value_bytes_whole"] - stats["value_bytes_touched"])
            stats["hbm_frac_step_touched"] = round(
                touched / (ms_per_step * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
            # each kernel reads the value tensor once: count its touched sectors
            untouched = stats["value_bytes_whole"] - stats["value_bytes_touched"]
            rl = result["roofline"]
            rl["bytes_per_launch_touched"] = nbytes[dom] - untouched
            rl["frac_touched"] = round((nbytes[dom] - untouched) / (dom_ms * 1e-3) / 1e9
                                       / peaks["hbm_gbs"], 4)
            if "fwd_alone" in result:
                fa = result["fwd_alone"]
                fa["frac_touched"] = round((nbytes["fused_forward"] - untouched)
                                           / (fa["fwd_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
        result["config"]["input_stats"] = stats
        if dom == "fused_backward":
            # the backward's own ceiling: its grad_value reductions (one float32
            # row of D channels per in-map corner) go through the L2's
            # reduction units, whose rate a reduction-only probe kernel
            # measured on B200: 6.4 TB/s of payload (red.global.add.v4.f32 at
            # random 128-byte rows of an L2-resident float32 array the size of
            # the encoder's grad_value; bulk reductions from shared memory
            # reach the same rate)
            red_bytes = stats["in_map_corners_per_sample"] * w.samples * w.D * 4
            ach = red_bytes / (bwd_ms * 1e-3) / 1e9
            result["roofline"]["l2_reduction"] = {
                "bytes_per_launch": int(red_bytes), "achieved": round(ach, 1), "ceiling": 6400.0,
                "unit": "GB/s", "frac": round(ach / 6400.0, 4),
                "ceiling_source": "reduction-only probe kernel on B200 (not part of this bench)"}
        if not args.no_e2e:
            result["e2e"] = _time_e2e(_pinned(x), step, make_outputs, flush, min(args.steps, 50),
                                      w.samples, dev, 7)
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(w, x, args.cpu_seconds)
            result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(
                w, x, result["cpu_baseline"], args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        line = json.dumps(result)
        print(line, flush=True)
        if args.out:
            with open(args.out, "a") as f:
                f.write(line + "\n")
    return result


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "source": "fallback"}


def _time_nonfused(msda, t, w, nbytes, flush, n, value, value_scale=None):
    """msda_forward / msda_backward (pre-computed locations and weights) on the
    same workload: per-launch device times (L2 flushed before each)."""
    import torch
    stream = torch.cuda.current_stream()
    args = (value, t["spatial_shapes"], t["level_start_index"], t["sampling_locations"],
            t["attention_weights"])
    out = torch.empty_like(t["grad_output"])
    gv = torch.empty(value.shape, dtype=torch.float32, device=value.device)
    gl = torch.empty_like(t["sampling_locations"])
    ga = torch.empty_like(t["attention_weights"])
    f, b = [], []
    for i in range(n + 3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.fill_(float(i))
        e[0].record(stream)
        msda.forward(*args, out=out, value_scale=value_scale)
        e[1].record(stream)
        msda.zero_grads(gv)
        flush.fill_(float(i + 1))
        e[2].record(stream)
        msda.backward(*args, t["grad_output"], grad_value=gv, grad_sampling_locations=gl,
                      grad_attention_weights=ga, accumulate=True, value_scale=value_scale)
        e[3].record(stream)
        if i >= 3:
            f.append(e)
    torch.cuda.synchronize()
    fwd = statistics.mean(e[0].elapsed_time(e[1]) for e in f)
    bwd = statistics.mean(e[2].elapsed_time(e[3]) for e in f)
    peak = _peaks()["hbm_gbs"]
    return {"fwd_ms": round(fwd, 5), "bwd_ms": round(bwd, 5),
            "fwd_hbm_frac": round(nbytes["forward"] / (fwd * 1e-3) / 1e9 / peak, 4),
            "bwd_hbm_frac": round(nbytes["backward"] / (bwd * 1e-3) / 1e9 / peak, 4),
            "fwd_gsamples_per_s": round(w.samples / (fwd * 1e-3) / 1e9, 4), "launches": n}


def _time_fwd(msda, t, o, flush, n, value, value_scale, order, nbytes, peaks):
    """msda_fused_forward alone (nothing beside it on the GPU, L2 flushed
    before each launch)."""
    import torch
    stream = torch.cuda.current_stream()
    ts = []
    for i in range(n + 3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        flush.fill_(float(i))
        e[0].record(stream)
        msda.fused_forward(value, t["spatial_shapes"], t["level_start_index"],
                           t["reference_points"], t["sampling_offsets"], t["attention_logits"],
                           out=o["out"], query_order=order, value_scale=value_scale)
        e[1].record(stream)
        if i >= 3:
            ts.append(e)
    torch.cuda.synchronize()
    ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ts)
    return {"fwd_ms": round(ms, 5), "launches": n,
            "frac": round(nbytes["fused_forward"] / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}


def _time_bwd(msda, t, o, flush, n, value, value_scale, order, merge):
    """msda_fused_backward alone (zero-fill outside the events, L2 flushed
    before each launch) with the given grad_value reduction path."""
    import torch
    stream = torch.cuda.current_stream()
    ts = []
    for i in range(n + 3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        msda.zero_grads(o["grad_value"], o["grad_reference_points"])
        flush.fill_(float(i))
        e[0].record(stream)
        msda.fused_backward(value, t["spatial_shapes"], t["level_start_index"],
                            t["reference_points"], t["sampling_offsets"], t["attention_logits"],
                            t["grad_output"], accumulate=True, grad_value=o["grad_value"],
                            grad_reference_points=o["grad_reference_points"],
                            grad_sampling_offsets=o["grad_sampling_offsets"],
                            grad_attention_logits=o["grad_attention_logits"],
                            query_order=order, value_scale=value_scale, merge_reductions=merge)
        e[1].record(stream)
        if i >= 3:
            ts.append(e)
    torch.cuda.synchronize()
    ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ts)
    return {"reductions": "merged" if merge and order is None else "direct",
            "bwd_ms": round(ms, 5), "launches": n}


def _capture_step(step, nev):
    """The step captured once into a CUDA graph (its second stream included,
    through the step's own fork and join events), after one more run on the
    capture stream."""
    import torch
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        step([torch.cuda.Event() for _ in range(nev)])  # once more on the capture stream
        torch.cuda.synchronize()
        # thread-local capture: calls other threads make meanwhile (a process
        # group's watchdog) neither break the capture nor fail
        with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
            step([torch.cuda.Event() for _ in range(nev)])
    stream.wait_stream(cap)
    return g


def _graph_steps(step, nev, flush, n, barrier, agree):
    """n replays of the step from a CUDA graph captured once (both streams),
    the L2 flushed before each outside the timed events, bracketed by a
    barrier and a synchronize like the launched steps; the replays' event
    times in ms, or None (on every rank) when the capture failed on any:
    agree(ok) returns whether it succeeded on all ranks."""
    import torch
    try:
        g = _capture_step(step, nev)
    except RuntimeError as e:
        print(f"CUDA graph capture failed ({e}); the launched steps stand", file=sys.stderr)
        g = None
    if not agree(g is not None):
        return None
    for i in range(3):
        flush.fill_(float(i))
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    barrier()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    for i, (a, b) in enumerate(evs):
        flush.fill_(float(i))
        a.record(cur)
        g.replay()
        b.record(cur)
    torch.cuda.synchronize()
    barrier()
    del g
    return [a.elapsed_time(b) for a, b in evs]


def _time_warm(w, step, n):
    """The same step back to back with no L2 flush between steps (warm L2)."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(n + 3)]
    for ev in evs:
        step(ev)
    torch.cuda.synchronize()
    ms = [e[0].elapsed_time(e[3]) for e in evs[3:]]
    med = float(np.median(ms))
    return {"ms_per_step_median": round(med, 5), "value": round(w.samples / (med * 1e-3) / 1e9, 4),
            "unit": UNIT, "steps": n}


def _input_stats(w: wl.Workload, x: wl.Inputs, max_queries: int = 4096) -> dict:
    """Share of samples whose bilinear footprint lies wholly / partly outside
    the level map, from the fused inputs (loc = ref + off / (W, H), pixel =
    loc * size - 0.5), over every k-th query (at most `max_queries` per batch
    image); and, for problems of up to 4 M samples, the distinct value bytes
    the forward touches (whole 32-byte sectors)."""
    stride = max(1, int(np.ceil(w.num_queries / max_queries)))
    ref = x.reference_points[:, ::stride].astype(np.float64)        # [B, q, 2]
    off = x.sampling_offsets[:, ::stride].astype(np.float64)        # [B, q, M, L, K, 2]
    hw = x.spatial_shapes.astype(np.float64)                        # [L, 2] (H, W)
    wh = hw[:, ::-1]                                                # (W, H)
    loc = ref[:, :, None, None, None, :] + off / wh[None, None, None, :, None, :]
    px = loc * wh[None, None, None, :, None, :] - 0.5
    lo = np.floor(px)
    size = wh[None, None, None, :, None, :]
    inside = (px > -1) & (px < size)
    full_out = ~(inside[..., 0] & inside[..., 1])
    any_out = ((lo < 0) | (lo + 1 > size - 1)).any(axis=-1)
    # corners the backward reduces into grad_value: the in-map corners of the
    # samples that are taken
    in_map = np.zeros(full_out.shape)
    for dy in (0, 1):
        for dx in (0, 1):
            cx, cy = lo[..., 0] + dx, lo[..., 1] + dy
            in_map += (cx >= 0) & (cx < size[..., 0]) & (cy >= 0) & (cy < size[..., 1])
    in_map[full_out] = 0
    out = {"samples_counted": int(full_out.size),
           "fully_outside": round(float(full_out.mean()), 4),
           "any_corner_outside": round(float(any_out.mean()), 4),
           "in_map_corners_per_sample": round(float(in_map.mean()), 4)}
    if w.samples <= (4 << 20):
        loc = (x.reference_points.astype(np.float64)[:, :, None, None, None, :]
               + x.sampling_offsets.astype(np.float64) / wh[None, None, None, :, None, :])
        px = loc * wh[None, None, None, :, None, :] - 0.5
        x0 = np.floor(px[..., 0]).astype(np.int64)
        y0 = np.floor(px[..., 1]).astype(np.int64)
        Wl = x.spatial_shapes[:, 1][None, None, None, :, None]
        Hl = x.spatial_shapes[:, 0][None, None, None, :, None]
        start = x.level_start_index[None, None, None, :, None]
        b = np.arange(w.B)[:, None, None, None, None]
        m = np.arange(w.M)[None, None, :, None, None]
        elt = {"f32": 4, "bf16": 2, "s8": 1, "e4m3": 1}[w.dtype]
        row_bytes = w.D * elt
        rows = []
        for dy in (0, 1):
            for dx in (0, 1):
                xi, yi = x0 + dx, y0 + dy
                ok = (xi >= 0) & (xi < Wl) & (yi >= 0) & (yi < Hl)
                key = (b * w.S + start + yi * Wl + xi) * w.M + m
                rows.append(np.broadcast_to(key, ok.shape)[ok])
        rows = np.unique(np.concatenate(rows))
        sectors = np.unique((rows[:, None] * row_bytes + np.arange(0, row_bytes, 32)[None, :]) // 32)
        out["value_bytes_touched"] = int(sectors.size * 32)
        out["value_bytes_whole"] = int(w.B * w.S * w.M * row_bytes)
    return out


def _time_e2e(hin, step, make_outputs, flush, n, samples, dev, nev):
    """The same step through the public API with host buffers: every step
    copies its inputs from pinned host memory (`hin`) to the device and all
    its results back to pinned host memory.  The copies run on their own
    streams with two sets of device buffers, so step i+1's input copy and
    step i-1's result copy overlap step i's kernels (the L2 flush still runs
    before every step's kernels).  Time = first input copy to last result
    copy, over n steps after two untimed ones."""
    import torch
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    sets = [({k: torch.empty_like(v, device=dev) for k, v in hin.items()}, make_outputs())
            for _ in range(2)]
    hout = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in sets[0][1].items()}
    h2d = sum(v.numel() * v.element_size() for v in hin.values())
    d2h = sum(v.numel() * v.element_size() for v in hout.values())

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def run(steps, first=None):
        done_comp, done_out = [None, None], [None, None]
        last = None
        for i in range(steps):
            din, dout = sets[i % 2]
            with torch.cuda.stream(s_in):
                if done_comp[i % 2] is not None:
                    s_in.wait_event(done_comp[i % 2])  # step i-2 has read these inputs
                if i == 0 and first is not None:
                    first.record(s_in)
                for k in hin:
                    din[k].copy_(hin[k], non_blocking=True)
                copied = ev()
                copied.record(s_in)
            comp.wait_event(copied)
            if done_out[i % 2] is not None:
                comp.wait_event(done_out[i % 2])  # step i-2's results are on the host
            flush.fill_(float(i))
            step([ev() for _ in range(nev)], din, dout)
            c = ev()
            c.record(comp)
            done_comp[i % 2] = c
            with torch.cuda.stream(s_out):
                s_out.wait_event(c)
                for k in hout:
                    hout[k].copy_(dout[k], non_blocking=True)
                last = ev()
                last.record(s_out)
                done_out[i % 2] = last
        return last

    run(2)
    torch.cuda.synchronize()
    start = ev()
    end = run(n, start)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / n
    return {"value": round(samples / (ms * 1e-3) / 1e9, 4), "unit": UNIT,
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": n, "copies": "pinned host buffers; input and result copies on their own streams, "
                                  "overlapping the neighbouring steps' kernels",
            "link_gbs": _link_bandwidth(hin, hout, sets[0][0], sets[0][1], s_in, s_out)}


def _link_bandwidth(hin, hout, din, dout, s_in, s_out, reps: int = 5) -> dict:
    """The host link alone, with the step's own buffers: GB/s of the input
    copies (host to device), of the result copies (device to host), and of
    both at once on their two streams (each direction's bytes over the
    common time), the medians of `reps` rounds: the ceiling the e2e leg's
    copies can reach."""
    import torch

    def timed(h2d: bool, d2h: bool) -> float:
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record()
            s_in.wait_event(a)
            s_out.wait_event(a)
            if h2d:
                with torch.cuda.stream(s_in):
                    for k in hin:
                        din[k].copy_(hin[k], non_blocking=True)
            if d2h:
                with torch.cuda.stream(s_out):
                    for k in hout:
                        hout[k].copy_(dout[k], non_blocking=True)
            torch.cuda.current_stream().wait_stream(s_in)
            torch.cuda.current_stream().wait_stream(s_out)
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e-3)
        return statistics.median(ts)

    nin = sum(v.numel() * v.element_size() for v in hin.values())
    nout = sum(v.numel() * v.element_size() for v in hout.values())
    t_in, t_out, t_both = timed(True, False), timed(False, True), timed(True, True)
    return {"h2d": round(nin / t_in / 1e9, 1), "d2h": round(nout / t_out / 1e9, 1),
            "both_h2d": round(nin / t_both / 1e9, 1), "both_d2h": round(nout / t_both / 1e9, 1)}


# ------------------------------------------------------- the oracle legs --

def _oracle_sample(w: wl.Workload, x: wl.Inputs, frac: float, block: int = 512):
    """About `frac` of the workload's queries in contiguous blocks of `block`
    queries spread evenly over the query axis (all levels stay represented,
    and each block keeps the access locality of a full pass), with the full
    value map: the inputs of a bounded oracle pass.  frac >= 1: every query."""
    Q = w.num_queries
    if frac >= 1.0 or block >= Q:
        qs = np.arange(Q)
    else:
        nblk = max(1, int(round(frac * Q / block)))
        starts = np.linspace(0, Q - block, nblk).astype(np.int64)
        qs = np.unique(np.concatenate([np.arange(s0, s0 + block) for s0 in starts]))
    return {
        "value": x.value_f64(), "grad_output": np.ascontiguousarray(x.grad_output_f64()[:, qs]),
        "spatial_shapes": x.spatial_shapes, "level_start_index": x.level_start_index,
        "reference_points": np.ascontiguousarray(x.reference_points[:, qs]),
        "sampling_offsets": np.ascontiguousarray(x.sampling_offsets[:, qs]),
        "attention_logits": np.ascontiguousarray(x.attention_logits[:, qs]),
        "samples": w.B * len(qs) * w.M * w.L * w.K, "queries": len(qs),
        "what": ("every query" if len(qs) == Q else
                 f"{len(qs)} of {Q} queries in contiguous blocks of {block}"),
    }


def _sample_fraction(oracle, w: wl.Workload, x: wl.Inputs, seconds: float, passes: int = 3) -> float:
    """Fraction of the workload's queries whose fused fwd+bwd the oracle runs
    `passes` times within about `seconds` (one timed probe on a small block)."""
    probe = _oracle_sample(w, x, min(1.0, 1024 / w.num_queries))
    t0 = time.perf_counter()
    _oracle_step(oracle, probe)
    per_query = (time.perf_counter() - t0) / probe["queries"]
    return min(1.0, seconds / passes / (per_query * w.num_queries))


def _oracle_step(oracle, smp):
    oracle.fused_forward(smp["value"], smp["spatial_shapes"], smp["level_start_index"],
                         smp["reference_points"], smp["sampling_offsets"], smp["attention_logits"])
    oracle.fused_backward(smp["value"], smp["spatial_shapes"], smp["level_start_index"],
                          smp["reference_points"], smp["sampling_offsets"],
                          smp["attention_logits"], smp["grad_output"])


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w: wl.Workload, x: wl.Inputs, seconds: float) -> dict:
    """The fp64 oracle (plain C loops, one thread), fused forward + backward on
    the whole workload when a few passes fit in `seconds`, else on contiguous
    blocks of its queries, timed on this host's cores."""
    import oracle
    oracle.build()
    smp = _oracle_sample(w, x, _sample_fraction(oracle, w, x, seconds))
    t0 = time.perf_counter()
    passes = 0
    while True:
        _oracle_step(oracle, smp)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    rate = smp["samples"] * passes / el
    return {"value": round(rate / 1e9, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{smp['what']} ({smp['samples']} samples) x {passes} passes of fused "
                      f"fwd+bwd, {el:.1f} s", "host_cpus": os.cpu_count(), "cpu_model": _cpu_model(),
            "full_step_ms_extrapolated": round(w.samples / rate * 1e3, 1)}


def _cpu_worker(job):
    """One process of the all-cores oracle leg: fused fwd+bwd over its slice
    of the sampled queries, `passes` times; returns (seconds, samples)."""
    folder, q0, q1, passes = job
    import oracle
    d = {k: np.load(os.path.join(folder, k + ".npy"), mmap_mode="r")
         for k in ("value", "grad_output", "spatial_shapes", "level_start_index",
                   "reference_points", "sampling_offsets", "attention_logits")}
    smp = {k: (np.ascontiguousarray(v[:, q0:q1]) if k in ("grad_output", "reference_points",
                                                         "sampling_offsets", "attention_logits")
               else v) for k, v in d.items()}
    B, _, M, _ = d["value"].shape
    L, K = d["sampling_offsets"].shape[3], d["sampling_offsets"].shape[4]
    t0 = time.perf_counter()
    for _ in range(passes):
        _oracle_step(oracle, smp)
    return time.perf_counter() - t0, passes * B * (q1 - q0) * M * L * K


def cpu_baseline_all_cores(w: wl.Workload, x: wl.Inputs, one_thread: dict, seconds: float) -> dict:
    """The same oracle, unchanged, in one process per host core (spawned), each
    on its own slice of the sampled queries; value = all samples / the slowest
    process's time.  The per-process grad_value sums are not combined (a
    reduction the timing leaves out)."""
    import multiprocessing as mp
    import tempfile
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    smp = _oracle_sample(w, x, min(1.0, _sample_fraction(oracle, w, x, seconds) * cores))
    nq = smp["queries"]
    nproc = max(1, min(cores, nq))
    rate1 = one_thread["value"] * 1e9
    per_proc_samples = smp["samples"] / nproc
    passes = max(1, int(np.ceil(seconds * rate1 / per_proc_samples)))
    with tempfile.TemporaryDirectory() as folder:
        for k in ("value", "grad_output", "spatial_shapes", "level_start_index",
                  "reference_points", "sampling_offsets", "attention_logits"):
            np.save(os.path.join(folder, k + ".npy"), smp[k])
        bounds = np.linspace(0, nq, nproc + 1).astype(int)
        jobs = [(folder, int(bounds[i]), int(bounds[i + 1]), passes) for i in range(nproc)]
        with mp.get_context("spawn").Pool(nproc) as pool:
            res = pool.map(_cpu_worker, jobs)
    slowest = max(t for t, _ in res)
    total = sum(n for _, n in res)
    return {"value": round(total / slowest / 1e9, 6), "unit": UNIT, "cores": nproc,
            "kind": "oracle",
            "sample": f"{smp['what']} split over {nproc} spawned processes x {passes} "
                      f"passes of fused fwd+bwd, slowest {slowest:.1f} s"}


def run_reference(args):
    """The reference arm: the oracle, as it stands, on the host cores, each
    step a bounded sample of the workload (rank 0 only)."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    w = wl.WORKLOADS[args.workload]
    x = wl.generate(w, with_nonfused=False)
    # size the per-step sample so that warm-up + steps stay within ~2 minutes:
    # the whole workload when it fits, else contiguous blocks of its queries
    frac = _sample_fraction(oracle, w, x, 120.0, passes=args.steps + args.warmup)
    smp = _oracle_sample(w, x, frac)
    for _ in range(args.warmup):
        _oracle_step(oracle, smp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(oracle, smp)
    el = time.perf_counter() - t0
    rate = smp["samples"] * args.steps / el
    value = rate / 1e9
    sample = f"{smp['what']} ({smp['samples']} samples) per step, fused fwd+bwd"
    result = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(w.samples / rate * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded SplitMix64 + Box-Muller draws (no dataset)",
        "config": {"workload": w.name, "B": w.B, "levels_HW": [list(l) for l in w.levels],
                   "Q": w.num_queries, "M": w.M, "D": w.D, "L": w.L, "K": w.K,
                   "step": "oracle fused_forward + fused_backward (fp64 C loops)",
                   "parallelism": "one host thread"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    line = json.dumps(result)
    print(line, flush=True)
    if args.out:
        with open(args.out, "a") as f:
            f.write(line + "\n")
    return result


# ------------------------------------------------------------ DCNv3 core --

def dcn_algorithmic_bytes(w: wl.DcnWorkload) -> dict:
    Ho, Wo = w.out_hw
    e = {"f32": 4, "bf16": 2, "s8": 1}[w.dtype]
    er = {"f32": 4, "bf16": 2, "s8": 2}[w.dtype]
    x = w.N * w.H * w.W * w.G * w.C
    rows = w.N * Ho * Wo * w.G * w.C
    off, mask = w.samples * 8, w.samples * 4
    fwd = x * e + off + mask + rows * er
    bwd = rows * er + x * e + off + mask + x * 4 + off + mask
    return {"dcn_forward": fwd, "dcn_backward": bwd, "quantize": x * 3 if w.dtype == "s8" else 0}


def _dcn_to_device(x: wl.DcnInputs, dev):
    import torch

    def val(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    return {"input": val(x.input), "offset": torch.from_numpy(x.offset).to(dev),
            "mask": torch.from_numpy(x.mask).to(dev), "grad_output": val(x.grad_output)}


def _dcn_band(w: wl.DcnWorkload, x: wl.DcnInputs, max_samples: int):
    """A bounded sample of the workload: the top band of input rows of image 0,
    with the offsets, masks and output gradients of the output rows it
    yields (the same layer on a shorter map)."""
    import oracle
    Ho, Wo = w.out_hw
    per_row = Wo * w.G * w.K
    rows_out = max(1, min(Ho, max_samples // per_row))
    hb = min(w.H, rows_out * w.stride[0])
    hob, _ = oracle.dcn_output_size(hb, w.W, w.kernel, w.stride, w.pad, w.dil)
    hob = max(0, min(hob, Ho))
    return dict(x=x.input_f64()[0:1, :hb], off=x.offset[0:1, :hob], mask=x.mask[0:1, :hob],
                gy=x.grad_output_f64()[0:1, :hob], samples=hob * per_row, rows=hb)


def _dcn_oracle_pass(w: wl.DcnWorkload, band) -> None:
    import oracle
    og = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dil=w.dil)
    oracle.dcn_forward(band["x"], band["off"], band["mask"], **og)
    oracle.dcn_backward(band["x"], band["off"], band["mask"], band["gy"], **og)


def _dcn_oracle_cpu(w: wl.DcnWorkload, x: wl.DcnInputs, seconds: float):
    """The oracle's DCNv3 core (fp64 C loops, one thread), forward + backward
    on a band of image 0 of about 2^18 samples, repeated for `seconds`.
    Returns (G samples/s, sample text)."""
    import oracle
    oracle.build()
    band = _dcn_band(w, x, 1 << 18)
    t0 = time.perf_counter()
    passes = 0
    while True:
        _dcn_oracle_pass(w, band)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    text = (f"input rows 0..{band['rows'] - 1} of image 0 of {w.N} ({band['samples']} samples) "
            f"x {passes} passes, {el:.1f} s")
    return band["samples"] * passes / el / 1e9, text


def run_dcn(args):
    """The DCNv3 core step: msda_dcn_forward || zero-fill -> msda_dcn_backward
    (INT8 input: msda_quantize_value_s8 first), same timing rules as the
    attention step."""
    import torch
    import torch.distributed as dist
    import scale_deformable_attention_msdeformattn_b200 as msda

    world, rank, local = _dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    base = wl.DCN_WORKLOADS[args.workload]
    w = dataclasses.replace(base, index=base.index + 1000 * rank) if rank else base
    x = wl.generate_dcn(w)
    t = _dcn_to_device(x, dev)
    N, H, W, G, C = w.N, w.H, w.W, w.G, w.C
    Ho, Wo = w.out_hw
    geo = dict(kernel=w.kernel, stride=w.stride, pad=w.pad, dilation=w.dil)
    int8 = w.dtype == "s8"
    q = torch.empty((N, H, W, G, C), dtype=torch.int8, device=dev) if int8 else None
    qs = torch.empty((N, G), dtype=torch.float32, device=dev) if int8 else None
    def make_outputs():
        return {"out": torch.empty((N, Ho, Wo, G, C), dtype=t["grad_output"].dtype, device=dev),
                "grad_input": torch.empty((N, H, W, G, C), dtype=torch.float32, device=dev),
                "grad_offset": torch.empty_like(t["offset"]),
                "grad_mask": torch.empty_like(t["mask"])}

    outputs = make_outputs()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=dev)

    def step(ev, tin=None, o=None):
        tin = tin or t
        o = o or outputs
        stream = torch.cuda.current_stream()
        ev[0].record(stream)
        inp = tin["input"]
        if int8:
            msda.quantize_value_s8(inp.flatten(1, 2), value_s8=q.flatten(1, 2), value_scale=qs)
            inp = q
        ev[4].record(stream)
        msda.dcn_forward(inp, tin["offset"], tin["mask"], out=o["out"], value_scale=qs, **geo)
        side.wait_event(ev[4])  # enqueued after the forward, whose CTAs take the SMs first
        with torch.cuda.stream(side):
            msda.zero_grads(o["grad_input"].flatten(1, 2))
            ev[5].record(side)
        ev[1].record(stream)
        stream.wait_event(ev[5])
        ev[2].record(stream)
        msda.dcn_backward(inp, tin["offset"], tin["mask"], tin["grad_output"],
                          grad_input=o["grad_input"], accumulate=True, value_scale=qs,
                          grad_offset=o["grad_offset"], grad_mask=o["grad_mask"], **geo)
        ev[3].record(stream)
        return o

    def events(n):
        return [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(n)]

    warm = events(args.warmup)
    for i in range(args.warmup):
        flush.fill_(float(i))
        step(warm[i])
    torch.cuda.synchronize()
    if msda.device_status() != 0:
        raise SystemExit("kernels reported a device check")
    evs = events(args.steps)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for i in range(args.steps):
        flush.fill_(float(i))
        step(evs[i])
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    graphms = _graph_steps(step, 6, flush, args.steps, lambda: dist.barrier() if world > 1 else None,
                           lambda ok: _all_ranks(ok, world, dev))
    clocks.stop()
    stepms = [e[0].elapsed_time(e[3]) for e in evs]
    graph_ok = graphms is not None
    if not graph_ok:
        args.headline, graphms = "launched", stepms
    l_total_ms, l_value = aggregate_over_ranks(float(sum(stepms)), w.samples, args.steps, world, dev)
    g_total_ms, g_value = aggregate_over_ranks(float(sum(graphms)), w.samples, args.steps, world, dev)
    if args.headline == "graph":
        total_ms, value, headms = g_total_ms, g_value, graphms
    else:
        total_ms, value, headms = l_total_ms, l_value, stepms
    result = None
    if rank == 0:
        peaks = _peaks()
        nb = dcn_algorithmic_bytes(w)
        fwd_ms = statistics.mean(e[4].elapsed_time(e[1]) for e in evs)
        bwd_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
        dom, dom_ms = ("dcn_backward", bwd_ms) if bwd_ms >= fwd_ms else ("dcn_forward", fwd_ms)
        achieved = nb[dom] / (dom_ms * 1e-3) / 1e9
        ms_per_step = total_ms / args.steps
        result = {
            "metric": METRIC + " (DCNv3 core workload)", "value": round(value, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"f32": "f32", "bf16": "bf16 input / f32 accumulate",
                      "s8": "int8 input (per image-group scale) / bf16 rows / f32 accumulate"}[w.dtype],
            "data": "synthetic: seeded SplitMix64 + Box-Muller draws (no dataset)",
            "config": {"workload": w.name, "N": N, "H": H, "W": W, "G": G, "C": C,
                       "kernel": list(w.kernel), "stride": list(w.stride), "pad": list(w.pad),
                       "dilation": list(w.dil), "offset_sigma_px": w.offset_sigma,
                       "samples_per_step_per_gpu": w.samples,
                       "step": ("msda_quantize_value_s8 -> " if int8 else "")
                       + "msda_dcn_forward || msda_zero_grads (second stream) -> msda_dcn_backward",
                       "l2": "flushed between steps (256 MiB write outside the timed events)",
                       "timing": ("the step replayed from a CUDA graph captured once (both streams), "
                                  "events around each replay" if args.headline == "graph" else
                                  "the step's calls launched one by one, events around each step"),
                       "parallelism": f"dp{world} (independent batch per GPU)"},
            "fwd_ms": round(fwd_ms, 5), "bwd_ms": round(bwd_ms, 5),
            "step_ms_p10_p50_p90": [round(float(np.percentile(headms, p)), 5) for p in (10, 50, 90)],
            **_other_timing(args.headline, graph_ok, args.steps, (l_value, l_total_ms, stepms),
                            (g_value, g_total_ms, graphms)),
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
                         "peak": peaks["hbm_gbs"], "peak_source": peaks["source"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "bytes_per_launch": nb[dom],
                         "traffic": (lambda tr: tr["bytes"] if tr and tr.get("csrc") == csrc_hash()
                                     else None)(NCU_TRAFFIC.get((dom, w.name)))},
            "gpu_launches": (3 + (3 if int8 else 0)) * args.steps,
            "clocks": clocks.summary(),
        }
        if not args.no_e2e and world == 1:
            hin = {k: v.cpu().pin_memory() for k, v in t.items()}
            result["e2e"] = _time_e2e(hin, step, make_outputs, flush, min(args.steps, 50), w.samples,
                                      dev, 6)
        if world == 1 and not args.no_cpu_baseline:
            rate, sample = _dcn_oracle_cpu(w, x, args.cpu_seconds)
            result["cpu_baseline"] = {"value": round(rate, 6), "unit": UNIT, "cores": 1,
                                      "kind": "oracle", "sample": sample}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        line = json.dumps(result)
        print(line, flush=True)
        if args.out:
            with open(args.out, "a") as f:
                f.write(line + "\n")
    return result


def run_dcn_reference(args):
    """Reference arm for a DCNv3 workload: the oracle's DCNv3 core on a band of
    image 0 per step, sized so that warm-up + steps end in about two minutes
    (rank 0 only)."""
    world, rank, _ = _dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    w = wl.DCN_WORKLOADS[args.workload]
    x = wl.generate_dcn(w)
    probe = _dcn_band(w, x, 1 << 14)
    t0 = time.perf_counter()
    _dcn_oracle_pass(w, probe)
    per_sample = (time.perf_counter() - t0) / max(1, probe["samples"])
    budget = 120.0 / (args.steps + args.warmup)
    band = _dcn_band(w, x, int(max(1, budget / per_sample)))
    for _ in range(args.warmup):
        _dcn_oracle_pass(w, band)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _dcn_oracle_pass(w, band)
    el = time.perf_counter() - t0
    value = band["samples"] * args.steps / el / 1e9
    sample = f"input rows 0..{band['rows'] - 1} of image 0 ({band['samples']} samples) per step"
    result = {"impl": "reference", "metric": METRIC + " (DCNv3 core workload)", "value": round(value, 6),
              "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
              "ms_per_step": round(w.samples / (value * 1e9) * 1e3, 3), "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "f64",
              "data": "synthetic: seeded SplitMix64 + Box-Muller draws (no dataset)",
              "config": {"workload": w.name, "step": "oracle dcn_forward + dcn_backward (fp64 C loops)",
                         "parallelism": "one host thread"},
              "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": sample},
              "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                      "d2h_bytes_per_step": 0}}
    line = json.dumps(result)
    print(line, flush=True)
    if args.out:
        with open(args.out, "a") as f:
            f.write(line + "\n")
    return result


# ------------------------------------------------------ the whole layer --

def run_layer(args):
    """One MSDeformAttn layer step (forward + backward through autograd) at
    the workload's shape, C = M * D: the library's layer (tensor-core
    value / output projections, fused query head, core) beside the same
    layer built from torch bf16 linear layers around the fused core (the
    offsets and logits then make a round trip through HBM).  L2 flushed
    before each step; CUDA events on the current stream; one GPU."""
    import torch
    import torch.nn.functional as F
    import scale_deformable_attention_msdeformattn_b200 as msda

    w = wl.WORKLOADS[args.workload]
    B, S, Q, M, D, L, K = w.B, w.S, w.num_queries, w.M, w.D, w.L, w.K
    C = M * D
    P = M * L * K
    dev = torch.device("cuda", 0)
    torch.manual_seed(0)
    shapes = torch.tensor(w.levels, dtype=torch.int64, device=dev)
    starts = torch.from_numpy(wl.level_start_index(w.levels)).to(dev)
    x = wl.generate(w, with_nonfused=False)
    ref = torch.from_numpy(x.reference_points).to(dev)
    layer = msda.MSDeformAttn(d_model=C, n_levels=L, n_heads=M, n_points=K).to(dev)
    with torch.no_grad():
        layer.sampling_offsets.weight.normal_(0.0, w.offset_sigma / C ** 0.5)
        layer.attention_weights.weight.normal_(0.0, w.logit_sigma / C ** 0.5)
    query = torch.randn(B, Q, C, device=dev, requires_grad=True)
    feats = torch.randn(B, S, C, device=dev, requires_grad=True)
    gy = torch.randn(B, Q, C, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def library_step():
        y = layer(query, ref, feats, shapes, starts)
        y.backward(gy)

    bf = torch.bfloat16

    def torch_linear_step():
        # the same layer with torch bf16 linear layers around the fused core
        value = F.linear(feats.to(bf), layer.value_proj.weight.to(bf), layer.value_proj.bias.to(bf))
        qb = query.to(bf)
        off = F.linear(qb, layer.sampling_offsets.weight.to(bf), layer.sampling_offsets.bias.to(bf))
        logit = F.linear(qb, layer.attention_weights.weight.to(bf), layer.attention_weights.bias.to(bf))
        core = msda.MSDeformAttnFusedFunction.apply(
            value.view(B, S, M, D), shapes, starts, ref, off.float().view(B, Q, M, L, K, 2),
            logit.float().view(B, Q, M, L * K))
        y = F.linear(core.reshape(B, Q, C), layer.output_proj.weight.to(bf), layer.output_proj.bias.to(bf))
        y.float().backward(gy)

    def time(step, n):
        evs = []
        for i in range(args.warmup + n):
            flush.fill_(float(i))
            for t in (query, feats):
                t.grad = None
            layer.zero_grad(set_to_none=True)
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record()
            step()
            e[1].record()
            if i >= args.warmup:
                evs.append(e)
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in evs]
        return statistics.median(ms), ms

    lib_ms, _ = time(library_step, args.steps)
    tl_ms, _ = time(torch_linear_step, args.steps)
    if msda.device_status() != 0:
        raise SystemExit("kernels reported an error")
    # HBM bytes between the heads and the core, per forward: the torch path
    # writes and reads the bf16 offsets + logits, then writes and reads their
    # float32 copies the core takes; the library's head writes float32
    # locations + attention weights once and the core reads them once
    head_torch = B * Q * 3 * P * (2 + 2 + 4 + 4)
    head_lib = B * Q * 3 * P * (4 + 4)
    line = {
        "metric": "MSDeformAttn layer fwd+bwd ms (projections, query head, core)",
        "value": round(lib_ms, 4), "unit": "ms", "higher_is_better": False,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "dtype": "bf16 operands / f32 accumulate (layer); core bf16 value",
        "data": "synthetic: seeded offsets / logits heads, random query and features",
        "config": {"workload": w.name, "B": B, "S": S, "Q": Q, "C": C, "M": M, "L": L, "K": K,
                   "l2": "flushed before each step"},
        "torch_linear_layer_ms": round(tl_ms, 4),
        "speedup_vs_torch_linear_layer": round(tl_ms / lib_ms, 3),
        "head_to_core_hbm_bytes": {"torch_linear_layer": head_torch, "library": head_lib,
                                   "avoided": head_torch - head_lib},
        "gpu": torch.cuda.get_device_name(0),
    }
    print(json.dumps(line), flush=True)
    if args.out:
        with open(args.out, "a") as f:
            f.write(json.dumps(line) + "\n")
    return line


def main(argv=None):
    args = parse_args(argv)
    dcn = args.workload in wl.DCN_WORKLOADS
    if args.layer:
        return run_layer(args)
    if args.impl == "reference":
        return run_dcn_reference(args) if dcn else run_reference(args)
    return run_dcn(args) if dcn else run_ours(args)


if __name__ == "__main__":
    main()
