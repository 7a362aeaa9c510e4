#!/usr/bin/env python
"""Benchmark of the RMM hot path (score -> select -> pack -> gemm) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload linear_4096] [--rho 0.5]

One step is one pass of the whole path over one synthetic input: the library's
C-ABI stage calls rmm_score, rmm_select, rmm_pack and rmm_gemm, which are the
kernels rmm_matmul_reduced chains. CUDA events bracket every stage on the
launching stream; L2 is flushed (256 MiB written, 256 MiB read) before every
timed step and
a short device-side sleep lets the host queue the whole step before the GPU
reaches it, so host launch overhead is not timed. The metric is effective
TFLOP/s on the kept FLOPs (2·M·N·k per product) and the speedup of the same
pipeline against rho = 1. With --gpus N (under torchrun) every rank runs an
independent replica of the workload (weak scaling, no collective on the data
path); timing is the max over ranks.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from input_adaptive_reduced_02_b200 import inputs, rmm  # noqa: E402

RHOS = (0.3, 0.5, 0.7, 0.9, 1.0)
METRIC = "reduced-matmul effective TFLOP/s (kept FLOPs 2*M*N*k) and speedup vs rho=1"
FLUSH_BYTES = 256 << 20
SLEEP_CYCLES = 1_000_000  # ~0.5-0.8 ms: lets the host queue a whole step ahead of the GPU
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "gemm_tc_linear_4096_rho0.5.txt")
GEMM_SOURCES = [os.path.join(ROOT, "input_adaptive_reduced_02_b200", "csrc", f)
                for f in ("gemm_tc.cu", "rmm_device.cuh")]


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="linear_4096",
                    choices=["linear_4096", "f32_64x256x64", "qk_32x4096x128", "pv_8192", "pv_16384", "pv_32768",
                             "pv_softmax_8192", "pv_softmax_16384", "pv_softmax_32768",
                             "mlp_up", "mlp_down", "decode_4096", "decode_mlp_up", "decode_mlp_up_m1",
                             "w8_linear_4096", "w8_decode_mlp_up_m1"])
    ap.add_argument("--rho", type=float, default=None, help="retention ratio of the headline step")
    ap.add_argument("--heads", type=int, default=32,
                    help="heads of the attention workloads (32 is the workload; fewer for small profiling runs)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the rho sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--score-mode", choices=["product", "a_only"], default="product",
                    help="slice score: ||A[:,k]||·||B[k,:]|| (library default) or the pages' ||A[:,k]||")
    ap.add_argument("--no-quality", action="store_true",
                    help="skip the error check of top-k against random selection")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- workloads
class Problem:
    """A batch of products A[b] (M×K) · B[b] (K×N) on the device."""

    def __init__(self, name, A, B, b_kmajor, out_dtype, rho, descr):
        self.name, self.A, self.B, self.b_kmajor = name, A, B, b_kmajor
        self.out_dtype, self.rho, self.descr = out_dtype, rho, descr
        self.mode = "product"
        A3 = A if A.dim() == 3 else A.unsqueeze(0)
        B3 = B if B.dim() == 3 else B.unsqueeze(0)
        self.batch, self.M, self.K = A3.shape
        self.N = B3.shape[1] if b_kmajor else B3.shape[2]
        self.b_norm = None  # B's cached norms: the step uses them (decode: B is a resident weight)
        self.scale = None   # INT8 weight: B holds the int8 codes, W = B · diag(scale)
        self.logits = None  # P·V with its softmax producer: the logits; A is the P the call writes
        # k = ceil(rho·K): the library's rmm_keep_count on the GPU arm; the CPU
        # reference arm substitutes the oracle's, so that it never loads librmm
        self.keep_count = rmm.keep_count

    @property
    def gemv(self):
        """Decode shape: the library streams B's kept rows without packing."""
        return self.M <= 16 and not self.b_kmajor

    @property
    def stream(self):
        """Narrow product (N <= 128, bf16): the library zeroes B's dropped rows
        and streams A whole through the GEMM instead of packing A (the route
        rule is the library's; a tensor without device memory counts as aligned)."""
        if self.scale is not None or self.gemv or self.logits is not None:
            return False
        A3 = self.A if self.A.dim() == 3 else self.A.unsqueeze(0)
        b, M, K = A3.shape
        lda = A3.stride(1) if M > 1 else K
        sA = A3.stride(0) if b > 1 else M * lda
        ptr = self.A.data_ptr() if self.A.is_cuda else 0
        dt = rmm.RMM_BF16 if self.A.dtype == torch.bfloat16 else rmm.RMM_F32
        return rmm.lib().rmm_fused_route(b, M, self.N, int(self.b_kmajor), dt, ctypes.c_void_p(ptr), lda,
                                         sA) == rmm.ROUTE_STREAM

    def k_keep(self, rho):
        return self.keep_count(rho, self.K)

    def kept_flops(self, rho):
        return 2.0 * self.batch * self.M * self.N * self.k_keep(rho)


def make_problem(name, device, seed, rho, heads=32):
    if name == "linear_4096":
        X, W = inputs.linear_projection(seed=seed, device=device)
        return Problem(name, X, W, False, torch.float32, rho or 0.5,
                       "X[4096x4096] bf16 (1% outlier channels x20) · W[4096x4096] bf16 N(0,0.02^2)")
    if name == "f32_64x256x64":
        A, B = inputs.lognormal_slices_f32(seed=seed, device=device)
        return Problem(name, A, B, False, torch.float32, rho or 0.5,
                       "A[64x256] · B[256x64] f32, log-normal slice scales")
    if name == "qk_32x4096x128":
        Q, Km = inputs.attention_qk(seed=seed, device=device)
        return Problem(name, Q, Km, True, torch.bfloat16, rho or 0.5,
                       "Q,K [32][4096][128] bf16 (4 channels x8), S = Q·K^T reduced over head_dim, bf16 out")
    if name.startswith("pv_softmax_"):
        S = int(name.split("_")[2])
        L, V = inputs.attention_logits(bh=heads, S=S, d=128, seed=seed, device=device)
        P = torch.zeros(heads, S, S, dtype=torch.bfloat16, device=device)
        p = Problem(name, P, V, False, torch.float32, rho or 0.5,
                    f"L [{heads}][{S}][{S}] bf16 logits 3·N(0,1) -> P = causal softmax (bf16, written by the call) · "
                    f"V [{heads}][{S}][128] bf16, reduced over keys, scored while P is written")
        p.logits = L
        return p
    if name.startswith("pv_"):
        S = int(name.split("_")[1])
        P, V = inputs.attention_pv(bh=heads, S=S, d=128, seed=seed, device=device)
        return Problem(name, P, V, False, torch.float32, rho or 0.5,
                       f"P [{heads}][{S}][{S}] causal softmax bf16 · V [{heads}][{S}][128] bf16, reduced over keys")
    if name == "mlp_up":
        X, W = inputs.mlp_up(seed=seed, device=device)
        return Problem(name, X, W, False, torch.float32, rho or 0.5,
                       "X[2048x8192] (0.5% outliers x20) · W[8192x28672] bf16 N(0,0.01^2)")
    if name == "decode_4096":
        X, W = inputs.linear_projection(M=16, seed=seed, device=device)
        p = Problem(name, X[:1].contiguous(), W, False, torch.float32, rho or 0.5,
                    "decode: x[1x4096] (1% outlier channels x20) · W[4096x4096] bf16, W's norms cached")
        p.b_norm = rmm.b_norms(W) if str(device) != "cpu" else None
        return p
    if name in ("decode_mlp_up", "decode_mlp_up_m1"):
        X, W = inputs.mlp_up(seed=seed, device=device)
        m = 1 if name.endswith("_m1") else 16
        p = Problem(name, X[:m].contiguous(), W, False, torch.float32, rho or 0.5,
                    f"decode: x[{m}x8192] (0.5% outliers x20) · W[8192x28672] bf16 N(0,0.01^2), W's norms cached")
        p.b_norm = rmm.b_norms(W) if str(device) != "cpu" else None
        return p
    if name in ("w8_linear_4096", "w8_decode_mlp_up_m1"):
        if name == "w8_linear_4096":
            X, _ = inputs.linear_projection(seed=seed, device=device)
            Wq, sc = inputs.int8_weight(4096, 4096, std=0.02, seed=seed + 1, device=device)
            descr = "X[4096x4096] bf16 (1% outliers x20) · INT8 W[4096x4096] with per-column scales, W's norms cached"
        else:
            X, _ = inputs.mlp_up(seed=seed, device=device)
            X = X[:1].contiguous()
            Wq, sc = inputs.int8_weight(8192, 28672, std=0.01, seed=seed + 1, device=device)
            descr = "decode: x[1x8192] · INT8 W[8192x28672] with per-column scales, W's norms cached"
        p = Problem(name, X, Wq, False, torch.float32, rho or 0.5, descr)
        p.scale = sc
        p.b_norm = rmm.b_norms_w8(Wq, sc) if str(device) != "cpu" else None
        return p
    if name == "mlp_down":
        X, W = inputs.mlp_down(seed=seed, device=device)
        return Problem(name, X, W, False, torch.float32, rho or 0.5,
                       "SiLU(N(0,1))[2048x28672] · W[28672x8192] bf16 N(0,0.01^2)")
    raise ValueError(name)


# ----------------------------------------------------------------- staged step
class Pipeline:
    """Device buffers for one problem and the staged C-ABI calls of one step."""

    def __init__(self, p: Problem, rho_max: float, force_pack: bool = False):
        self.p = p
        self.stream = p.stream and not force_pack  # force_pack: the pack route's stage calls, for comparison
        dev = p.A.device
        kmax = p.k_keep(rho_max)
        kp = rmm.padded_keep(kmax)
        shp = (lambda r, c: (p.batch, r, c)) if p.A.dim() == 3 else (lambda r, c: (r, c))
        self.s = torch.empty((p.batch, p.K) if p.A.dim() == 3 else (p.K,), dtype=torch.float32, device=dev)
        self.idx_store = torch.empty(p.batch * kmax, dtype=torch.int32, device=dev)
        if p.logits is not None:  # softmax producer: row stats, then P and the scores in one pass
            self.a_store = None
            self.stats = torch.empty(p.batch, p.M, 2, dtype=torch.float32, device=dev)
            self.b_mask = torch.empty(shp(p.K, rmm.packed_b_ld(p.N)), dtype=p.A.dtype, device=dev)
        elif self.stream:  # B with its dropped rows zeroed; A is read as it is
            self.a_store = None
            self.b_mask = torch.empty(shp(p.K, rmm.packed_b_ld(p.N)), dtype=p.A.dtype, device=dev)
        else:
            self.a_store = torch.empty(p.batch * p.M * kp, dtype=p.A.dtype, device=dev)
            self.b_store = torch.empty(p.batch * kp * max(p.N, rmm.packed_b_ld(p.N)), dtype=p.A.dtype, device=dev)
        self.C = torch.empty(shp(p.M, p.N), dtype=p.out_dtype, device=dev)
        self.status = rmm.status_word(dev)

    def views(self, rho):
        p = self.p
        k = p.k_keep(rho)
        if self.stream or p.logits is not None:
            idx = self.idx_store[: p.batch * k].view(p.batch, k) if p.A.dim() == 3 else self.idx_store[:k]
            return k, idx, None, None
        kp = rmm.padded_keep(k)
        bshape = rmm.packed_b_shape(p.A.dim() == 3, p.batch, p.N, kp, p.b_kmajor)
        nb = 1
        for d in bshape:
            nb *= d
        B_S = self.b_store[:nb].view(bshape)
        if p.A.dim() == 3:
            idx = self.idx_store[: p.batch * k].view(p.batch, k)
            A_S = self.a_store[: p.batch * p.M * kp].view(p.batch, p.M, kp)
        else:
            idx = self.idx_store[:k]
            A_S = self.a_store[: p.M * kp].view(p.M, kp)
        return k, idx, A_S, B_S

    def step(self, rho, ev=None, breakdown=False):
        """One pass of score -> select -> pack -> gemm.

        ev: events to record. With breakdown, 5 events bracket every stage
        (the events break programmatic-launch overlap between stages);
        otherwise 3 events: before score, and immediately before and after
        the GEMM kernel itself."""
        p = self.p
        k, idx, A_S, B_S = self.views(rho)
        if ev:
            ev[0].record()
        if p.logits is not None:  # the producer writes P and the key scores
            rmm.softmax_row_stats(p.logits, out=self.stats, status=self.status)
            rmm.softmax_score(p.logits, self.stats, p.B if p.mode == "product" else None, P=p.A, s=self.s,
                              status=self.status)
        elif p.b_norm is not None:
            rmm.score_b_norms(p.A, p.b_norm, out=self.s, status=self.status)
        else:
            rmm.score(p.A, p.B, p.mode, p.b_kmajor, out=self.s, status=self.status)
        if ev and breakdown:
            ev[1].record()
        rmm.select(self.s, k, out=idx, status=self.status)
        if ev and breakdown:
            ev[2].record()
        if p.gemv:  # decode shape: no pack; the GEMV reads B's kept rows through idx
            if ev and breakdown:
                ev[3].record()
            elif ev:
                ev[1].record()
            if p.scale is not None:
                rmm.gemv_gather_w8(p.A, p.B, p.scale, idx, out=self.C)
            else:
                rmm.gemv_gather(p.A, p.B, idx, out=self.C)
            if ev:
                ev[4 if breakdown else 2].record()
            return
        if self.stream or p.logits is not None:  # B's dropped rows zeroed, then the GEMM over all of A
            rmm.mask_rows(p.B, idx, out=self.b_mask)
        elif p.scale is not None:
            rmm.pack_w8(p.A, p.B, p.scale, idx, out=(A_S, B_S), status=self.status)
        else:
            rmm.pack(p.A, p.B, idx, p.b_kmajor, out=(A_S, B_S), status=self.status)
        if ev and breakdown:
            ev[3].record()
        elif ev:
            # the library records these immediately around the GEMM kernel
            # (after the split-K zeroing kernel rmm_gemm may launch first)
            rmm.set_gemm_events(ev[1], ev[2])
        if p.logits is not None:  # P is causal: tiles stop at their last row's keys
            rmm.gemm_full(p.A, self.b_mask, p.N, out=self.C, status=self.status, causal_off=p.K - p.M)
        elif self.stream:
            rmm.gemm_full(p.A, self.b_mask, p.N, out=self.C, status=self.status)
        else:
            rmm.gemm(A_S, B_S, k, b_kmajor=p.b_kmajor, N=p.N, out=self.C, status=self.status)
        if ev and breakdown:
            ev[4].record()
        elif ev:
            rmm.set_gemm_events(None, None)


STAGES = ("score", "select", "pack", "gemm")


def step_descr(p) -> str:
    """What one timed step launches, by route (the stage names of stages_ms
    follow STAGES whatever the route: 'pack' is the masking of B's dropped
    rows on the stream route, 'score' the softmax producer when P is written)."""
    if p.logits is not None:
        return ("one rmm_pv_softmax_reduced call (row statistics, P written with the key scores, select, "
                "V's dropped rows zeroed, causal GEMM over P: 5 kernels)")
    # decode shapes whose score needs only x: the selection scores x itself
    folded = p.gemv and p.M <= 4 and p.K <= 8192
    if p.scale is not None:
        if p.gemv:
            return ("one rmm_matmul_reduced_w8 call with W's norms cached ("
                    + ("select scoring x itself, INT8 gather-GEMV: 2 kernels)" if folded
                       else "score, select, INT8 gather-GEMV: 3 kernels)"))
        return "one rmm_matmul_reduced_w8 call with W's norms cached (score, select, INT8 pack, gemm: 4 kernels)"
    if p.gemv:
        return ("one rmm_matmul_reduced_b_norms call ("
                + ("select scoring x itself, gather-GEMV: 2 kernels)" if folded
                   else "score of x, select, gather-GEMV: 3 kernels)"))
    if p.stream:
        return "one rmm_matmul_reduced call, stream route (score, select, B's dropped rows zeroed, gemm over A: 4 kernels)"
    if p.b_kmajor:
        return "one rmm_matmul_reduced call (score, select, pack of A's columns, pack of Kmat's columns, gemm: 5 kernels)"
    return "one rmm_matmul_reduced call (score, select, pack, gemm: 4 kernels)"


class Fused:
    """The one-call public path: rmm_matmul_reduced into a preallocated C with a
    reusable workspace (sized for rho_max). With b_norm, the call with B's
    norms cached (rmm_matmul_reduced_b_norms; the norms are computed once,
    outside the timed steps, as a caller would for a weight)."""

    def __init__(self, p: Problem, rho_max: float, b_norm=None):
        self.p = p
        dev = p.A.device
        self.C = torch.empty((p.batch, p.M, p.N) if p.A.dim() == 3 else (p.M, p.N), dtype=p.out_dtype, device=dev)
        if p.logits is not None:
            nb = rmm.pv_softmax_workspace_size(p.batch, p.M, p.K, p.N, p.k_keep(rho_max))
        else:
            nb = rmm.workspace_size_for(p.batch, p.M, p.K, p.N, p.k_keep(rho_max), p.A.dtype, p.b_kmajor)
        self.ws = rmm.Workspace(nb, dev)
        self.b_norm = b_norm if b_norm is not None else p.b_norm

    def step(self, rho, ev=None, breakdown=False):
        p = self.p
        if ev:
            ev[0].record()
        if p.logits is not None:
            rmm.pv_softmax_reduced(p.logits, p.B, rho, mode=p.mode, P=p.A, out=self.C, workspace=self.ws)
        elif p.scale is not None:
            rmm.matmul_reduced_w8(p.A, p.B, p.scale, rho, b_norm=p.b_norm, mode=p.mode, out=self.C,
                                  workspace=self.ws)
        elif self.b_norm is not None:
            rmm.matmul_reduced_b_norms(p.A, p.B, self.b_norm, rho, out=self.C, workspace=self.ws,
                                       b_kmajor=p.b_kmajor)
        else:
            rmm.matmul_reduced(p.A, p.B, rho, p.mode, out=self.C, workspace=self.ws, b_kmajor=p.b_kmajor)
        if ev:
            ev[1].record()


class Unfused:
    """P·V with its softmax producer done in two library calls: the producer
    writes P alone, then rmm_pv_reduced scores P by reading it back, selects,
    and multiplies (what the fused call saves is that read of P)."""

    def __init__(self, p: Problem, rho: float):
        self.p = p
        dev = p.A.device
        self.stats = torch.empty(p.batch, p.M, 2, dtype=torch.float32, device=dev)
        self.C = torch.empty(p.batch, p.M, p.N, dtype=p.out_dtype, device=dev)
        self.ws = None

    def step(self, rho, ev=None, breakdown=False):
        p = self.p
        if ev:
            ev[0].record()
        rmm.softmax_row_stats(p.logits, out=self.stats)
        rmm.softmax_score(p.logits, self.stats, score=False, P=p.A)
        _, self.ws = rmm.pv_reduced(p.A, p.B, rho, p.mode, out=self.C, workspace=self.ws)
        if ev:
            ev[1].record()


class L2Flush:
    """Writes a 256 MiB buffer (evicting everything from the 126 MB L2), then
    reads a second one so that the dirty lines are written back before the
    timed step starts and the step finds a cold, clean L2."""

    def __init__(self, device):
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def timed_steps(pipe, rho: float, steps: int, flush, breakdown=False):
    """Run `steps` steps (L2 flushed and the host queued ahead before each).

    Returns (per-step ms, per-stage ms lists). For the staged Pipeline without
    breakdown the stages are {"pre_gemm": score+select+pack, "gemm": gemm};
    for the Fused call {"call": the whole call}."""
    fused = isinstance(pipe, (Fused, Dense, Unfused))
    n_ev = 2 if fused else (5 if breakdown else 3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    for i in range(steps):
        flush()
        torch.cuda._sleep(SLEEP_CYCLES)
        pipe.step(rho, evs[i], breakdown)
    torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[-1]) for e in evs]
    names = ("call",) if fused else (STAGES if breakdown else ("pre_gemm", "gemm"))
    stage_ms = {s: [e[j].elapsed_time(e[j + 1]) for e in evs] for j, s in enumerate(names)}
    return step_ms, stage_ms


class Dense:
    """The dense product of the same shapes through torch (cuBLAS bf16/f32),
    timed like the step: context for the reduced call, not part of it."""

    def __init__(self, p: Problem):
        self.p = p
        B = p.B
        if p.scale is not None:
            B = (B.float() * p.scale[None, :]).to(torch.bfloat16)
        self.B = B.transpose(-1, -2) if p.b_kmajor else B
        self.C = None

    def step(self, rho, ev=None, breakdown=False):
        if ev:
            ev[0].record()
        self.C = torch.matmul(self.p.A, self.B)
        if ev:
            ev[1].record()


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report it, keep going
            self.err = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                util = self.nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, util, r))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        busy = [s for s in self.samples if s[1] > 0] or self.samples
        bits = 0
        for s in busy:
            bits |= s[2]
        names = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[0] for s in busy) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(busy)}


# ----------------------------------------------------------------- roofline helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gemm_source_hash():
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the GEMM from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    kv = {}
    with open(PROFILE_TRAFFIC) as f:
        for line in f:
            if ":" in line and not line.lstrip().startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != gemm_source_hash():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------- CPU oracle timing
def oracle_cpu_timing(p: Problem, rho: float, budget_s: float, max_steps: int):
    """Time the fp64 oracle on the workload (rank 0 host cores): whole steps
    while they fit the budget, else the batch items (heads) it completes,
    scaled to the step (said in `sample`)."""
    from oracle import rmm_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count()
    mode = O.SCORE_A_ONLY if p.mode == "a_only" else O.SCORE_PRODUCT

    def f64(t):
        return t.to("cpu", torch.float32).numpy().astype(np.float64)

    def item(b):
        """The oracle's inputs for batch item b, converted when needed."""
        A = p.A[b] if p.A.dim() == 3 else p.A
        B = p.B[b] if p.B.dim() == 3 else p.B
        if p.logits is not None:
            return f64(p.logits[b][None]), f64(B[None])
        B64 = O.dequantize_w8(B.to("cpu").numpy(), p.scale.to("cpu").numpy()) if p.scale is not None else f64(B)
        return f64(A), (B64.T if p.b_kmajor else B64)

    def run(a, b):
        if p.logits is not None:
            O.pv_softmax_reduced(a, b, rho, mode)
        else:
            O.matmul_reduced(a, b, rho, mode)

    steps, items, t_items = 0, 0, 0.0
    t_start = time.perf_counter()
    while steps < max_steps:
        done = 0
        for b in range(p.batch):
            a, bb = item(b)
            t0 = time.perf_counter()
            run(a, bb)
            t_items += time.perf_counter() - t0
            done += 1
            items += 1
            if time.perf_counter() - t_start > budget_s:
                break
        if done == p.batch:
            steps += 1
        if time.perf_counter() - t_start > budget_s:
            break
    if items == 0:
        return None
    t = t_items / items * p.batch  # seconds per whole step
    sample = (f"{steps} full step(s)" if items % p.batch == 0 and steps else
              f"{items} of {p.batch} batch items timed, scaled to the step (extrapolated)")
    return {"value": p.kept_flops(rho) / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{sample} of {p.name} at rho={rho} (fp64 NumPy oracle: "
                      f"{'softmax, ' if p.logits is not None else ''}score, top-k, reduced product), "
                      f"{t * 1e3:.1f} ms per step"}


# ----------------------------------------------------------------- arms
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not torch.distributed.is_initialized():
        backend = "nccl" if args.impl == "ours" else "gloo"
        kw = {"timeout": datetime.timedelta(seconds=300)}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device(f"cuda:{local}")
        torch.distributed.init_process_group(backend, **kw)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over the ranks (a no-op for one rank)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(step_ms_local_total: float, steps: int, flops_per_rank_step: float, world: int):
    """Whole-job throughput of `world` replicas: every rank processed its own
    steps; the job took as long as the slowest rank. Returns (ms per step,
    TFLOP/s over all ranks)."""
    total = max_over_ranks(step_ms_local_total, world)
    ms = total / steps
    return ms, world * flops_per_rank_step / (ms * 1e-3) / 1e12


def run_reference(args):
    # The oracle needs no device and no collective: rank 0 runs it, the other
    # ranks of a torchrun launch exit at once.
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from oracle import rmm_oracle as O
    name = args.workload
    p = make_problem(name, "cpu", 0, args.rho, heads=args.heads)
    p.keep_count = O.keep_count
    p.mode = args.score_mode
    rho = p.rho
    budget = 150.0
    res = oracle_cpu_timing(p, rho, budget_s=budget, max_steps=max(1, args.steps))
    line = {"impl": "reference", "metric": METRIC,
            "value": res["value"] if res else None, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": 0, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": name, "descr": p.descr, "batch": p.batch, "M": p.M,
                                              "K": p.K, "N": p.N, "rho": rho, "k_keep": p.k_keep(rho),
                                              "score_mode": p.mode,
                                              "out_dtype": str(p.out_dtype).replace("torch.", "")},
            "cpu_baseline": res,
            "e2e": {"value": res["value"] if res else None, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_ours(args):
    rank, world, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device(f"cuda:{local}")
    p = make_problem(args.workload, dev, seed=rank, rho=args.rho, heads=args.heads)
    p.mode = args.score_mode
    rho = p.rho
    rho_max = rho if args.no_sweep else 1.0
    call = Fused(p, rho_max)
    pipe = Pipeline(p, rho_max)
    flush = L2Flush(dev)

    with ClockSampler(local) as clocks:
        for _ in range(max(3, args.warmup)):
            call.step(rho)
        rmm.check(call.ws)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        n0 = rmm.launch_count()
        t_wall0 = time.perf_counter()
        step_ms, _ = timed_steps(call, rho, args.steps, flush)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        wall_s = time.perf_counter() - t_wall0
        launches = rmm.launch_count() - n0
        rmm.check(call.ws)
        # the same step through the four stage calls, with events around the
        # GEMM launch: the dominant kernel's duration for the roofline
        for _ in range(3):
            pipe.step(rho)
        staged_ms, stage_ms = timed_steps(pipe, rho, args.steps, flush)
        rmm.check(pipe.status)
    clk = clocks.summary()

    ms_per_step, value = job_throughput(sum(step_ms), args.steps, p.kept_flops(rho), world)

    # rho sweep: the fused call (and the GEMM inside the staged pipeline), speedup against rho = 1
    sweep = {}
    if not args.no_sweep and p.K > 1:
        n = max(10, args.steps // 2)
        for r in RHOS:
            for _ in range(3):
                call.step(r)
                pipe.step(r)
            sm, _ = timed_steps(call, r, n, flush)
            _, st = timed_steps(pipe, r, n, flush)
            sweep[r] = {"ms": statistics.median(sm), "gemm_ms": statistics.median(st["gemm"]),
                        "k_keep": p.k_keep(r)}
        t1 = sweep[1.0]["ms"]
        for r in RHOS:
            d = sweep[r]
            d["speedup_vs_rho1"] = t1 / d["ms"]
            d["effective_tflops"] = p.kept_flops(r) / (d["ms"] * 1e-3) / 1e12
            d["gemm_tflops"] = p.kept_flops(r) / (d["gemm_ms"] * 1e-3) / 1e12
        rmm.check(call.ws)
        rmm.check(pipe.status)
        sweep = {f"{r:g}": {k: (round(v, 4) if isinstance(v, float) else v) for k, v in d.items()}
                 for r, d in sweep.items()}

    # P·V with its softmax producer: the same work in two calls (P written, then
    # read back by rmm_pv_reduced to be scored), timed the same way
    unfused = None
    if p.logits is not None:
        uf = Unfused(p, rho)
        for _ in range(3):
            uf.step(rho)
        ums, _ = timed_steps(uf, rho, max(5, args.steps), flush)
        u_ms = statistics.median(ums)
        unfused = {"ms": round(u_ms, 5), "fused_speedup": round(u_ms / statistics.median(step_ms), 4),
                   "calls": "rmm_softmax_row_stats + rmm_softmax_score (P only) + rmm_pv_reduced (reads P to score)"}
        del uf
        torch.cuda.empty_cache()

    # the stream route against the pack route it replaces (stage calls score,
    # select, pack, GEMM), same inputs, same timing
    pack_ref = None
    if p.stream and not args.no_sweep:
        pk = Pipeline(p, rho, force_pack=True)
        for _ in range(3):
            pk.step(rho)
        pms, _ = timed_steps(pk, rho, max(5, args.steps), flush)
        rmm.check(pk.status)
        p_ms = statistics.median(pms)
        pack_ref = {"ms": round(p_ms, 5), "stream_route_speedup": round(p_ms / statistics.median(step_ms), 4),
                    "calls": "rmm_score + rmm_select + rmm_pack + rmm_gemm (A packed)"}
        del pk
        torch.cuda.empty_cache()

    # the dense product of the same shapes (cuBLAS through torch), for context
    dense = None
    if not args.no_sweep:
        dn = Dense(p)
        for _ in range(3):
            dn.step(1.0)
        dms, _ = timed_steps(dn, 1.0, max(10, args.steps // 2), flush)
        d_ms = statistics.median(dms)
        dense = {"ms": round(d_ms, 5), "impl": "torch.matmul (cuBLAS), dense over all K",
                 "reduced_call_speedup": {r: round(d_ms / v["ms"], 4) for r, v in sweep.items()}}
        del dn
        torch.cuda.empty_cache()

    gemm_ms_timed = statistics.mean(stage_ms["gemm"])
    # per-stage breakdown (separate pass: events between stages cost the overlap)
    _, bd = timed_steps(pipe, rho, max(10, args.steps // 2), flush, breakdown=True)
    stage_mean = {s: statistics.mean(v) for s, v in bd.items()}
    rmm.check(pipe.status)
    del pipe, call
    torch.cuda.empty_cache()

    # the same call with B's norms cached (a weight's norms are computed once)
    cached = None
    if p.mode == "product" and p.b_norm is None and p.logits is None:
        bn = rmm.b_norms(p.B, p.b_kmajor)
        ccall = Fused(p, rho, b_norm=bn)
        for _ in range(3):
            ccall.step(rho)
        cms, _ = timed_steps(ccall, rho, max(10, args.steps // 2), flush)
        rmm.check(ccall.ws)
        cached = {"ms": round(statistics.median(cms), 5),
                  "effective_tflops": round(p.kept_flops(rho) / (statistics.median(cms) * 1e-3) / 1e12, 3),
                  "note": "rmm_matmul_reduced_b_norms with ||B[k,:]|| from rmm_b_norms computed once "
                          "outside the timed steps; the score then reads A only"}
        del ccall, bn
        torch.cuda.empty_cache()

    quality = None if args.no_quality else quality_check(p, rho, seed=rank)

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(p, rho, max(5, min(20, args.steps)), world)

    peaks, peak_src = measured_peaks()
    gemm_ms_max = max_over_ranks(gemm_ms_timed, world)
    dominant = max(stage_mean, key=stage_mean.get)
    # the dominant kernel's duration is taken from the timed region itself
    roof_ms = dict(stage_mean)
    if dominant == "gemm":
        roof_ms["gemm"] = gemm_ms_timed
    roof = roofline(p, rho, roof_ms, dominant, peaks, peak_src)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_cpu_timing(p, rho, budget_s=15.0, max_steps=20)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if p.A.dtype == torch.bfloat16 else "f32",
            "data": "synthetic",
            "config": {"workload": p.name, "descr": p.descr, "batch": p.batch, "M": p.M, "K": p.K, "N": p.N,
                       "rho": rho, "k_keep": p.k_keep(rho), "score_mode": p.mode,
                       "out_dtype": str(p.out_dtype).replace("torch.", ""),
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed before every timed step (256 MiB written, then another 256 MiB read)",
                       "step": step_descr(p),
                       "timing": "CUDA events on the launching stream around each call; a device sleep before "
                                 "each step hides host launch overhead. The GEMM's duration for the roofline "
                                 "comes from a second timed loop of the same step made of the four stage "
                                 "calls, with events before and after the GEMM launch; the stage breakdown "
                                 "from a third pass with events between all stages"},
            "step_ms_spread": {"min": round(min(step_ms), 5), "median": round(statistics.median(step_ms), 5),
                               "max": round(max(step_ms), 5)},
            "stages_ms": {s: round(v, 5) for s, v in stage_mean.items()},
            "stages_gbs": stage_gbs(p, rho, stage_mean),
            "cached_b_norm_call": cached,
            "quality": quality,
            "staged_region_ms": {"step": round(statistics.mean(staged_ms), 5),
                                 "pre_gemm": round(statistics.mean(stage_ms["pre_gemm"]), 5),
                                 "gemm": round(gemm_ms_timed, 5)},
            "wall_s_timed_region": round(wall_s, 4),
            "gemm_ms_max_over_ranks": round(gemm_ms_max, 5),
            "roofline": roof,
            "sweep": sweep,
            "dense_reference": dense,
            "unfused_reference": unfused,
            "pack_route_reference": pack_ref,
            "e2e": e2e,
            "gpu_launches": int(launches),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def stage_bytes(p: Problem, rho):
    """Algorithmic HBM bytes of each stage for one step (all batch items)."""
    k = p.k_keep(rho)
    kp = rmm.padded_keep(k)
    eb = p.A.element_size()
    ob = torch.tensor([], dtype=p.out_dtype).element_size()
    wb = 1 if p.scale is not None else eb  # bytes per element of B as stored (INT8 codes)
    b_read = 0 if (p.mode == "a_only" or p.b_norm is not None) else p.K * p.N * wb
    ldb = p.N if p.b_kmajor else rmm.packed_b_ld(p.N)
    if p.logits is not None:
        # producer: the visible logits twice (row statistics, then P), P written
        # whole, V read; GEMM: P's key blocks up to each 256-row tile's last row
        ldm = rmm.packed_b_ld(p.N)
        off = p.K - p.M
        vis = sum(min(p.K, q + 1 + off) for q in range(p.M))
        tiles = sum(min(256, p.M - m0) * min(p.K, -(-(min(p.M, m0 + 256) + off) // 64) * 64)
                    for m0 in range(0, p.M, 256))
        return {
            "score": (2 * vis * eb + p.M * p.K * 2 + p.K * p.N * eb + 8 * p.M + 4 * p.K) * p.batch,
            "select": (4 * p.K + 4 * k) * p.batch,
            "pack": (k * p.N * eb + p.K * ldm * eb) * p.batch,
            "gemm": (tiles * 2 + p.K * ldm * eb + p.M * p.N * ob) * p.batch,
        }
    if p.stream:  # mask: k rows of B read, K rows written; GEMM: all of A, B_M and C
        ldm = rmm.packed_b_ld(p.N)
        return {
            "score": (p.M * p.K * eb + b_read + 4 * p.K) * p.batch,
            "select": (4 * p.K + 4 * k) * p.batch,
            "pack": (k * p.N * eb + p.K * ldm * eb) * p.batch,
            "gemm": (p.M * p.K * eb + p.K * ldm * eb + p.M * p.N * ob) * p.batch,
        }
    if p.gemv:  # no pack; the GEMV reads k rows of B, k columns of A, writes C
        return {
            "score": (p.M * p.K * eb + b_read + 4 * p.K) * p.batch,
            "select": (4 * p.K + 4 * k) * p.batch,
            "pack": 0,
            "gemm": (k * p.N * wb + p.M * k * eb + 4 * k + p.M * p.N * ob) * p.batch,
        }
    return {
        "score": (p.M * p.K * eb + b_read + 4 * p.K) * p.batch,
        "select": (4 * p.K + 4 * k) * p.batch,
        "pack": (p.M * p.K * eb + k * p.N * wb + p.M * kp * eb + kp * ldb * eb) * p.batch,
        "gemm": ((p.M + p.N) * kp * eb + p.M * p.N * ob) * p.batch,
    }


def stage_gbs(p: Problem, rho, stage_mean):
    by = stage_bytes(p, rho)
    return {s: round(by[s] / (stage_mean[s] * 1e-3) / 1e9, 1) for s in stage_mean if by[s] > 0}


NEAR_TIE_REL = 1e-5  # relative score window around the k-th largest inside which the parity tests accept swaps


def quality_check(p: Problem, rho, seed):
    """Relative Frobenius error against the dense product (torch f32 matmul on
    the GPU, a measurement reference only) of the library's top-k selection and
    of a seeded random selection of the same size (the pages' baseline), both
    through the library's pack and GEMM; first batch item only."""
    A = p.A[0] if p.A.dim() == 3 else p.A
    B = p.B[0] if p.B.dim() == 3 else p.B
    k = p.k_keep(rho)
    Bf = (B.t() if p.b_kmajor else B).float()
    if p.scale is not None:
        Bf = Bf * p.scale[None, :]
    dense = A.float() @ Bf
    nd = torch.linalg.norm(dense).item()
    idx = torch.empty(k, dtype=torch.int32, device=A.device)
    g = torch.Generator(device=A.device)
    g.manual_seed(1000 + seed)
    ridx = torch.randperm(p.K, generator=g, device=A.device)[:k].sort().values.to(torch.int32).contiguous()
    if p.scale is not None:
        bn = p.b_norm if p.b_norm is not None else rmm.b_norms_w8(B, p.scale)
        C, _ = rmm.matmul_reduced_w8(A, B, p.scale, rho, b_norm=bn, mode=p.mode, idx_out=idx)
        if p.gemv:
            Cr = rmm.gemv_gather_w8(A, B, p.scale, ridx)
        else:
            A_S, B_S = rmm.pack_w8(A, B, p.scale, ridx)
            Cr = rmm.gemm(A_S, B_S, k, N=p.N)
    else:
        C, _ = rmm.matmul_reduced(A, B, rho, p.mode, torch.float32, idx_out=idx, b_kmajor=p.b_kmajor)
        A_S, B_S = rmm.pack(A, B, ridx, p.b_kmajor)
        Cr = rmm.gemm(A_S, B_S, k, b_kmajor=p.b_kmajor, N=p.N)
    # the selection's shape: slices whose score lies within the parity tests'
    # near-tie window of the k-th largest (where a rounding-order difference may
    # swap kept and dropped slices), and how contiguous the kept indices are
    if p.mode == "a_only":
        s = rmm.score(A, None, "a_only")
    elif p.b_norm is not None or p.scale is not None:
        s = rmm.score_b_norms(A, p.b_norm if p.b_norm is not None else rmm.b_norms_w8(B, p.scale))
    else:
        s = rmm.score(A, B, p.mode, b_kmajor=p.b_kmajor)
    s = s.reshape(-1)[:p.K].double()
    t = torch.topk(s, k).values[-1].item()
    in_window = int((torch.abs(s - t) <= NEAR_TIE_REL * t).sum().item())
    runs = 1 + int((torch.diff(idx.long()) != 1).sum().item()) if k > 1 else 1
    torch.cuda.synchronize()
    e_top = torch.linalg.norm(C - dense).item() / nd
    e_rand = torch.linalg.norm(Cr - dense).item() / nd
    return {"rel_fro_err_topk": round(e_top, 6), "rel_fro_err_random": round(e_rand, 6),
            "score_mode": p.mode, "item": 0, "reference": "dense f32 product (torch matmul on the GPU)",
            "selection": {"kept": k, "threshold_score": t, "near_tie_window_rel": NEAR_TIE_REL,
                          "slices_in_window": in_window, "kept_runs": runs, "kept_per_run": round(k / runs, 3)}}


def roofline(p: Problem, rho, stage_mean, dominant, peaks, peak_src):
    k = p.k_keep(rho)
    eb = p.A.element_size()
    ob = torch.tensor([], dtype=p.out_dtype).element_size()
    gemm_bytes = stage_bytes(p, rho)["gemm"]
    ridge = (peaks["bf16_tflops"] * 1e12) / (peaks["hbm_gbs"] * 1e9)
    if dominant == "gemm" and (p.gemv or p.A.dtype == torch.bfloat16) and p.kept_flops(rho) / gemm_bytes < ridge:
        # below the ridge (P·V, Q·Kᵀ's output write): the GEMM is bound by HBM
        ach = gemm_bytes / (stage_mean["gemm"] * 1e-3) / 1e9
        return {"kernel": "gemv_gather_kernel" if p.gemv else "gemm_tc_kernel", "bound": "hbm",
                "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None,
                "algorithmic_bytes_per_launch": gemm_bytes,
                "bytes_note": ("stream route: all of A (its kept columns reach nearly every 32-byte sector), "
                               "B with dropped rows zeroed, C" if p.stream else "kept operands and C"),
                "arithmetic_intensity": round(p.kept_flops(rho) / gemm_bytes, 1), "ridge": round(ridge, 1),
                "peak_source": f"{peak_src} HBM copy bandwidth"}
    if dominant == "gemm" and p.M >= 128 and p.N >= 128:
        flops = p.kept_flops(rho)
        ach = flops / (stage_mean["gemm"] * 1e-3) / 1e12
        peak = peaks["bf16_tflops"] if p.A.dtype == torch.bfloat16 else None
        traffic = recorded_traffic() if p.name == "linear_4096" and abs(rho - 0.5) < 1e-12 else None
        return {"kernel": "gemm_tc_kernel", "bound": "tensor", "achieved": round(ach, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(ach / peak, 4) if peak else None, "traffic": traffic,
                "algorithmic_flops_per_launch": flops,
                "peak_source": f"{peak_src} bf16 dense burst (cuBLAS)" if peak else "n/a (f32 CUDA-core path)"}
    # bandwidth-bound stage: algorithmic bytes per launch
    by = stage_bytes(p, rho)[dominant]
    ach = by / (stage_mean[dominant] * 1e-3) / 1e9
    return {"kernel": dominant, "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None, "algorithmic_bytes_per_launch": by,
            "peak_source": f"{peak_src} HBM copy bandwidth"}


def run_e2e(p: Problem, rho, steps, world):
    """Same metric through the public fused call with pinned host buffers:
    H2D of A and B, rmm_matmul_reduced, D2H of C, all inside the timed region."""
    resident_b = p.b_norm is not None  # decode: the weight and its norms stay on the device
    hA = p.A.to("cpu").pin_memory()
    hB = None if resident_b else p.B.to("cpu").pin_memory()
    dA = torch.empty_like(p.A)
    dB = p.B if resident_b else torch.empty_like(p.B)
    shape = (p.batch, p.M, p.N) if p.A.dim() == 3 else (p.M, p.N)
    dC = torch.empty(shape, dtype=p.out_dtype, device=p.A.device)
    hC = torch.empty(shape, dtype=p.out_dtype).pin_memory()

    def call(ws=None):
        if p.scale is not None:
            return rmm.matmul_reduced_w8(dA, dB, p.scale, rho, b_norm=p.b_norm, mode=p.mode, out=dC, workspace=ws)
        if resident_b:
            return rmm.matmul_reduced_b_norms(dA, dB, p.b_norm, rho, out=dC, workspace=ws)
        return rmm.matmul_reduced(dA, dB, rho, p.mode, out=dC, workspace=ws, b_kmajor=p.b_kmajor)

    dA.copy_(p.A)
    if not resident_b:
        dB.copy_(p.B)
    _, ws = call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dA.copy_(hA, non_blocking=True)
        if not resident_b:
            dB.copy_(hB, non_blocking=True)
        call(ws)
        hC.copy_(dC, non_blocking=True)
        e1.record()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    rmm.check(ws)
    ms = max_over_ranks(statistics.mean(ts), world)
    return {"value": round(world * p.kept_flops(rho) / (ms * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(hA.numel() * hA.element_size()
                                      + (0 if hB is None else hB.numel() * hB.element_size())),
            "d2h_bytes_per_step": int(hC.numel() * hC.element_size())}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
