"""Host-side checks of bench.py that need no GPU: the whole-job aggregation over
ranks (two gloo ranks on the CPU, as under torchrun) and the reference arm,
which times the fp64 oracle on the host."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_totals, out_q):
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, tflops = bench.job_throughput(local_totals[rank], 10, 2e12, world)
        out_q.put((rank, ms, tflops))
    finally:
        dist.destroy_process_group()


def test_job_throughput_is_the_slowest_rank_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    totals = [10.0, 20.0]  # ms for 10 steps on each rank
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, totals, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tflops in results:
        assert ms == pytest.approx(2.0)  # the slower rank: 20 ms / 10 steps
        assert tflops == pytest.approx(2 * 2e12 / 2e-3 / 1e12)  # both ranks' work over that time


def test_reference_arm_times_the_oracle_on_the_host():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2", "--warmup", "0",
                        "--workload", "f32_64x256x64"], cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "f32_64x256x64" and line["config"]["k_keep"] == 128


def test_reference_arm_follows_the_score_mode():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--workload", "f32_64x256x64", "--score-mode", "a_only"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"]["score_mode"] == "a_only" and line["value"] > 0

