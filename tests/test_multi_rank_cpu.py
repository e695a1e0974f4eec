"""The multi-GPU path is "replicas only": every rank runs the same per-GPU workload on its own
weights and the job time is the max over ranks.  This checks that host logic with two gloo ranks
on the CPU (no GPU, no NCCL)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import tq_inputs as I


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each replica draws its own weights
        w = I.weights(16, 64, I.seed_for(1, 0, 0) + bench.rank_seed_offset(rank))
        gathered = [torch.zeros_like(w) for _ in range(world)]
        dist.all_gather(gathered, w)
        distinct = not torch.equal(gathered[0], gathered[1])
        # per-rank step times: the job time is the slowest rank
        ms = 2.0 + rank
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        value = bench.weak_scaling_value(1_000_000_000, world, ms_max)
        out.put((rank, distinct, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, distinct, ms_max, value in res:
        assert distinct
        assert ms_max == 3.0                       # max over ranks, not the local time
        assert value == pytest.approx(2e9 / 3e-3 / 1e9)  # both ranks' bytes over the slowest time


def test_single_rank_aggregation():
    assert bench.max_over_ranks(1.5, 1) == 1.5
    assert bench.weak_scaling_value(6_530_000_000, 1, 1000.0) == pytest.approx(6.53)


def test_reference_arm_json_line():
    # `bench.py --impl reference` runs the CPU oracle on the host (no GPU) and prints one JSON
    # line with the GPU arm's metric and config plus the reference-arm keys
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--cpu-seconds", "0.3"], cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3 and d["ms_per_step"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "Llama-3-8B" in d["config"]["workload"]
