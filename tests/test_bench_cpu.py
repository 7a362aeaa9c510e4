"""Host-side checks of bench.py that need no GPU: the whole-job aggregation over
ranks (two gloo ranks on the CPU, as under torchrun), the reference arm, which
times the fp64 oracle on the host, and the roofline arithmetic (algorithmic
bytes per stage, bound chosen by arithmetic intensity) on shape-only tensors."""
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


def test_reference_arm_never_loads_the_library():
    """The reference arm runs the oracle alone: its process maps no librmm.so
    (k comes from the oracle's keep_count, not the library's)."""
    code = ("import sys, json; sys.argv = ['bench.py']; import bench; "
            "bench.main(['--impl', 'reference', '--steps', '1', '--warmup', '0', '--workload', 'f32_64x256x64']); "
            "print(json.dumps({'maps_librmm': 'librmm.so' in open('/proc/self/maps').read()}))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": "", "PYTHONPATH": ROOT})
    assert r.returncode == 0, r.stderr[-2000:]
    last = json.loads(r.stdout.strip().splitlines()[-1])
    assert last == {"maps_librmm": False}


def test_reference_arm_follows_the_score_mode():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--workload", "f32_64x256x64", "--score-mode", "a_only"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"]["score_mode"] == "a_only" and line["value"] > 0



# ---------------------------------------------------------------- roofline arithmetic
PEAKS = {"hbm_gbs": 6548.2, "bf16_tflops": 1652.0}


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def _meta(bench, name, a_shape, b_shape, dtype, b_kmajor=False, out=None):
    import torch
    A = torch.empty(a_shape, dtype=dtype, device="meta")
    B = torch.empty(b_shape, dtype=dtype, device="meta")
    return bench.Problem(name, A, B, b_kmajor, out or torch.float32, 0.5, "")


def test_stage_bytes_of_the_linear_workload():
    """Algorithmic bytes per stage at 4096³, rho 0.5 (k = 2048, bf16 in, f32 out)."""
    import torch
    bench = _bench()
    p = _meta(bench, "linear_4096", (4096, 4096), (4096, 4096), torch.bfloat16)
    by = bench.stage_bytes(p, 0.5)
    n = 4096
    assert by["score"] == 2 * n * n * 2 + 4 * n             # A and W read once, scores written
    assert by["select"] == 4 * n + 4 * 2048                 # scores read, indices written
    assert by["pack"] == n * n * 2 + 3 * n * 2048 * 2 == 83886080  # A whole, W's kept rows, A_S and B_S
    assert by["gemm"] == 2 * n * 2048 * 2 + n * n * 4       # A_S, B_S, f32 C


def test_roofline_bound_follows_arithmetic_intensity():
    import torch
    bench = _bench()
    # tensor-bound GEMM: 2·4096·4096·2048 flops in 62.7 us
    p = _meta(bench, "linear_4096", (4096, 4096), (4096, 4096), torch.bfloat16)
    r = bench.roofline(p, 0.5, {"gemm": 0.0627}, "gemm", PEAKS, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 2 * 4096 * 4096 * 2048 / 62.7e-6 / 1e12) < 0.01
    assert abs(r["frac"] - r["achieved"] / 1652.0) < 1e-4
    # decode GEMV (M = 1, W's norms cached): HBM-bound on the kept rows of W
    p = _meta(bench, "decode_mlp_up_m1", (1, 8192), (8192, 28672), torch.bfloat16)
    p.b_norm = object()
    r = bench.roofline(p, 0.5, {"gemm": 0.056}, "gemm", PEAKS, "measured")
    assert r["bound"] == "hbm" and r["kernel"] == "gemv_gather_kernel"
    assert r["algorithmic_bytes_per_launch"] == 4096 * 28672 * 2 + 4096 * 2 + 4 * 4096 + 28672 * 4 == 235020288
    assert abs(r["achieved"] - 235020288 / 56e-6 / 1e9) < 0.1
    # P·V (32 heads, S 16384, d 128): below the ridge, HBM-bound
    p = _meta(bench, "pv_16384", (32, 16384, 16384), (32, 16384, 128), torch.bfloat16)
    r = bench.roofline(p, 0.5, {"gemm": 3.0}, "gemm", PEAKS, "measured")
    assert r["bound"] == "hbm" and r["arithmetic_intensity"] < r["ridge"]
    # ... on the stream route: all of P, V with its dropped rows zeroed, O in f32
    assert p.stream and r["bytes_note"].startswith("stream route")
    assert r["algorithmic_bytes_per_launch"] == 32 * (16384 * 16384 * 2 + 16384 * 128 * 2 + 16384 * 128 * 4)
    # Q·Kᵀ (B = Kᵀ given K-major, bf16 out): the output write keeps it below the ridge
    p = _meta(bench, "qk_32x4096x128", (32, 4096, 128), (32, 4096, 128), torch.bfloat16, b_kmajor=True,
              out=torch.bfloat16)
    r = bench.roofline(p, 0.5, {"gemm": 0.3}, "gemm", PEAKS, "measured")
    assert r["bound"] == "hbm" and r["arithmetic_intensity"] < r["ridge"]
    # a memory-bound stage as the dominant one reports its own bytes
    p = _meta(bench, "linear_4096", (4096, 4096), (4096, 4096), torch.bfloat16)
    r = bench.roofline(p, 0.5, {"pack": 0.02}, "pack", PEAKS, "measured")
    assert r["bound"] == "hbm" and r["algorithmic_bytes_per_launch"] == 83886080


def test_step_description_follows_the_route():
    """The bench line's config.step names the kernels a step launches on each
    route (shape-only problems: no device memory needed)."""
    import torch
    bench = _bench()
    p = _meta(bench, "linear_4096", (4096, 4096), (4096, 4096), torch.bfloat16)
    assert "4 kernels" in bench.step_descr(p) and "pack" in bench.step_descr(p)
    p = _meta(bench, "decode_mlp_up_m1", (1, 8192), (8192, 28672), torch.bfloat16)
    assert "gather-GEMV: 2 kernels" in bench.step_descr(p)
    p = _meta(bench, "decode_mlp_up", (16, 8192), (8192, 28672), torch.bfloat16)
    assert "gather-GEMV: 3 kernels" in bench.step_descr(p)
    p = _meta(bench, "pv_16384", (32, 16384, 16384), (32, 16384, 128), torch.bfloat16)
    assert p.stream and "stream route" in bench.step_descr(p)
    p = _meta(bench, "qk_32x4096x128", (32, 4096, 128), (32, 4096, 128), torch.bfloat16, b_kmajor=True,
              out=torch.bfloat16)
    assert "5 kernels" in bench.step_descr(p)
