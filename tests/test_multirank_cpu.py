"""Host logic of multi-GPU runs, exercised with gloo ranks on the CPU: the
weak-scaling workload split, the max-over-ranks timing, the ranks'
agreement on the CUDA-graph timing, and the reference arm under torchrun
(only rank 0 reports).  No GPU is used."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from scale_deformable_attention_msdeformattn_b200 import workloads as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(wl.WORKLOADS["tiny_f32"], rank)
        total, value = bench.aggregate_over_ranks(times[rank], w.samples, 10, world)
        # the graph-capture agreement: false on every rank if false on any
        agreed = (bench._all_ranks(True, world), bench._all_ranks(rank == 0, world))
        out[rank] = (total, value, w.seed, agreed)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_split():
    world = 2
    port = _free_port()
    times = [3.0, 5.0]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    samples = 1 * 16 * 2 * 2 * 2  # tiny workload: B*Q*M*L*K
    for r in range(world):
        total, value, seed, agreed = res[r]
        assert total == 5.0  # the slowest rank sets the time
        assert abs(value - world * samples * 10 / 5e-3 / 1e9) < 1e-12
        assert agreed == (True, False)  # a capture failed on one rank: every rank falls back
    assert res[0][2] != res[1][2]  # every rank draws its own batch


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_reports_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--workload", "tiny_f32"]
    res = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT, timeout=280)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "G samples/s"
    for key in ("metric", "value", "steps", "warmup", "ms_per_step", "higher_is_better", "cpu_baseline",
                "e2e", "config"):
        assert key in d
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
