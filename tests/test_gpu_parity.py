"""GPU parity: every stage of the CUDA path (through the C ABI) against the fp64
oracle, on seeded inputs at sizes the oracle finishes in seconds that still
span several tiles and ragged tails, plus the edge cases of the method."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O
from input_adaptive_reduced_02_b200 import inputs, rmm

from _parity import (check_product, check_scores, check_selection, check_single, f64, product_tol)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ab(M, K, N, dtype, seed, outlier=True):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    A = torch.randn(M, K, generator=g, device=DEV)
    B = torch.randn(K, N, generator=g, device=DEV)
    if outlier:
        A *= torch.exp(torch.randn(K, generator=g, device=DEV))[None, :]
        B *= torch.exp(torch.randn(K, generator=g, device=DEV))[:, None]
    return A.to(dtype).contiguous(), B.to(dtype).contiguous()


SHAPES = [
    (300, 1000, 520),   # ragged M and N tiles, k_pad > k_keep
    (129, 257, 257),    # one row / column past a tile, odd K (scalar score and pack paths)
    (200, 300, 100),    # N <= 128: 128-wide tensor-core tiles
    (1, 40, 1),         # single row / column
    (5, 7, 3),          # K < 32
    (257, 64, 517),     # N not a multiple of 4: direct-store epilogue
    (384, 512, 768),    # exact tiles
]


@pytest.fixture(params=[2, 1], ids=["cta_pair", "one_sm"])
def gemm_cta_group(request):
    prev = rmm.set_gemm_cta_group(request.param)
    yield request.param
    rmm.set_gemm_cta_group(prev)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_stages_match_oracle(shape, dtype, gemm_cta_group):
    if dtype == torch.float32 and gemm_cta_group == 1:
        pytest.skip("the f32 path does not use the tensor-core GEMM")
    M, K, N = shape
    A, B = _ab(M, K, N, dtype, seed=M * 7 + K)
    A64, B64 = f64(A), f64(B)
    for mode in ("product", "a_only"):
        s = rmm.score(A, B, mode)
        check_scores(s.cpu().numpy(), O.slice_scores(A64, B64, mode))
        for rho in (0.3, 0.5, 1.0):
            k = O.keep_count(rho, K)
            assert rmm.keep_count(rho, K) == k
            idx = rmm.select(s, k)
            # integer stage: bit-exact against the oracle's selection on the same f32 scores
            assert idx.cpu().numpy().tolist() == O.select_top(s.cpu().numpy(), k).tolist()
            kp = rmm.padded_keep(k)
            ii = idx.long()
            # B given row-major: kept rows copied as they are (N-major operand)
            A_S, B_S = rmm.pack(A, B, idx)
            assert A_S.shape == (M, kp) and B_S.shape == (kp, rmm.packed_b_ld(N))
            assert torch.equal(A_S[:, :k], A[:, ii]) and torch.equal(B_S[:k, :N], B[ii, :])
            assert not A_S[:, k:].any() and not B_S[k:].any() and not B_S[:, N:].any()
            # B given as Bᵀ (the Kmat form): kept columns, K-major operand
            Bt = B.t().contiguous()
            A_S2, B_St = rmm.pack(A, Bt, idx, b_kmajor=True)
            assert torch.equal(A_S2, A_S) and B_St.shape == (N, kp)
            assert torch.equal(B_St[:, :k], Bt[:, ii]) and not B_St[:, k:].any()
            for out_dtype in (torch.float32, torch.bfloat16):
                tol = product_tol(dtype, out_dtype)
                C = rmm.gemm(A_S, B_S, k, out_dtype, N=N)
                check_product(C, A64, B64, idx.cpu().numpy(), tol)
                C2 = rmm.gemm(A_S2, B_St, k, out_dtype, b_kmajor=True)
                check_product(C2, A64, B64, idx.cpu().numpy(), tol)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("rho", [0.3, 0.5, 0.7, 1.0])
def test_fused_matmul_reduced(dtype, rho, gemm_cta_group):
    A, B = _ab(300, 1000, 520, dtype, seed=11)
    k = rmm.keep_count(rho, 1000)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, B, rho, "product", torch.float32, idx_out=idx)
    rmm.check(ws)
    check_single(A, B, rho, "product", C, idx)


def test_config_f32_64x256x64_end_to_end():
    A, B = inputs.lognormal_slices_f32(64, 256, 64, seed=0, device=DEV)
    idx = torch.empty(128, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, B, 0.5, "product", torch.float32, idx_out=idx)
    rmm.check(ws)
    nb, err = check_single(A, B, 0.5, "product", C, idx)
    assert err <= 1e-5


def test_batched_qk_small(gemm_cta_group):
    Q, Km = inputs.attention_qk(bh=3, S=300, d=128, seed=1, device=DEV)
    Q = Q[:, :200].contiguous()  # S_q != S_k
    k = rmm.keep_count(0.5, 128)
    idx = torch.empty(3, k, dtype=torch.int32, device=DEV)
    S, ws = rmm.qk_reduced(Q, Km, 0.5, out_dtype=torch.float32, idx_out=idx)
    rmm.check(ws)
    for h in range(3):
        check_single(Q[h], Km[h], 0.5, "product", S[h], idx[h], b_kmajor=True)
    S16, _ = rmm.qk_reduced(Q, Km, 0.5, out_dtype=torch.bfloat16, workspace=ws)
    for h in range(3):
        check_product(S16[h], f64(Q[h]), f64(Km[h]).T, idx[h].cpu().numpy(), 1e-2)


def test_batched_pv_small(gemm_cta_group):
    P, V = inputs.attention_pv(bh=2, S=700, d=128, seed=2, device=DEV)
    for rho in (0.3, 0.5, 0.7):
        k = rmm.keep_count(rho, 700)
        idx = torch.empty(2, k, dtype=torch.int32, device=DEV)
        Oo, ws = rmm.pv_reduced(P, V, rho, idx_out=idx)
        rmm.check(ws)
        for h in range(2):
            check_single(P[h], V[h], rho, "product", Oo[h], idx[h])


def test_ties_go_to_lower_index_and_zero_slices_last():
    # duplicated columns give exactly equal f32 scores on both sides
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    base = torch.randn(70, 9, generator=g, device=DEV)
    A = base[:, torch.arange(90, device=DEV) % 9].contiguous()  # 10 copies of each of 9 columns
    A[:, 3::17] = 0.0                                            # some zero columns
    B = torch.ones(90, 33, device=DEV)
    A, B = A.to(torch.bfloat16), B.to(torch.bfloat16)
    s = rmm.score(A, B)
    s_ref = O.slice_scores(f64(A), f64(B))
    check_scores(s.cpu().numpy(), s_ref)
    for rho in (0.1, 0.35, 0.5, 0.9, 0.99):
        k = O.keep_count(rho, 90)
        idx = rmm.select(s, k)
        # exact ties in both precisions: the selections must be identical
        assert idx.cpu().numpy().tolist() == O.select_top(s_ref, k).tolist()


def test_extreme_keep_counts():
    A, B = _ab(100, 300, 90, torch.bfloat16, seed=21)
    for rho in (1e-9, 1.0):
        k = rmm.keep_count(rho, 300)
        assert k == (1 if rho < 1 else 300)
        idx = torch.empty(k, dtype=torch.int32, device=DEV)
        C, ws = rmm.matmul_reduced(A, B, rho, idx_out=idx)
        rmm.check(ws)
        check_single(A, B, rho, "product", C, idx)


def test_empty_rows_still_select():
    A = torch.zeros(0, 50, dtype=torch.bfloat16, device=DEV)
    B = torch.randn(50, 20, device=DEV).to(torch.bfloat16)
    idx = torch.full((25,), -1, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, B, 0.5, idx_out=idx)
    rmm.check(ws)
    assert C.shape == (0, 20)
    # every score is 0, so the tie rule keeps the lowest 25 indices
    assert idx.cpu().tolist() == list(range(25))


def test_determinism_bit_identical():
    A, B = _ab(300, 1000, 520, torch.bfloat16, seed=31)
    outs = []
    for _ in range(2):
        s = rmm.score(A, B)
        idx = rmm.select(s, 500)
        C, _ = rmm.matmul_reduced(A, B, 0.5)
        outs.append((s.clone(), idx.clone(), C.clone()))
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def test_strided_inputs():
    # rows of A and B taken from wider buffers (ld > cols)
    A0, B0 = _ab(130, 600, 300, torch.bfloat16, seed=41)
    A = A0[:, :512]
    B = B0[:512, :264]
    assert A.stride(0) == 600 and B.stride(0) == 300
    idx = torch.empty(rmm.keep_count(0.5, 512), dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, B, 0.5, idx_out=idx)
    rmm.check(ws)
    check_single(A.contiguous(), B.contiguous(), 0.5, "product", C, idx)


def test_nonfinite_is_reported():
    A, B = _ab(64, 128, 64, torch.bfloat16, seed=51)
    A[3, 17] = float("nan")
    C, ws = rmm.matmul_reduced(A, B, 0.5)
    with pytest.raises(rmm.RMMError) as e:
        rmm.check(ws)
    assert e.value.status == rmm.RMM_ERR_NONFINITE
    # the status word was cleared; a clean call reports OK
    A[3, 17] = 0.0
    rmm.matmul_reduced(A, B, 0.5, workspace=ws)
    rmm.check(ws)


def test_launch_counter_counts_kernels():
    A, B = _ab(64, 128, 64, torch.bfloat16, seed=61)
    n0 = rmm.launch_count()
    rmm.matmul_reduced(A, B, 0.5)
    torch.cuda.synchronize()
    # score (one launch for A's and B's norms), select, pack (A's columns and B's rows in one launch), gemm
    assert rmm.launch_count() - n0 == 4


@pytest.mark.parametrize("batch", [1, 3])
def test_split_k_tiles_zeroed_inside_the_select_launch(batch, gemm_cta_group):
    """A shape whose last GEMM round is split along K (f32 C): in the fused call
    the select launch's spare blocks zero those C tiles, so no separate zeroing
    kernel runs; C is filled with NaN first, so a tile left unzeroed shows."""
    M, K, N = 2048, 512, 1024
    g = torch.Generator(device=DEV)
    g.manual_seed(71 + batch)
    A = torch.randn(batch, M, K, generator=g, device=DEV).to(torch.bfloat16)
    B = torch.randn(batch, K, N, generator=g, device=DEV).to(torch.bfloat16)
    out = torch.full((batch, M, N), float("nan"), device=DEV)
    idx = torch.empty(batch, rmm.keep_count(0.5, K), dtype=torch.int32, device=DEV)
    n0 = rmm.launch_count()
    C, ws = rmm.matmul_reduced(A, B, 0.5, out=out, idx_out=idx)
    torch.cuda.synchronize()
    rmm.check(ws)
    assert rmm.launch_count() - n0 == 4  # score, select (+ zeroing), pack (A and B), gemm
    for b in range(batch):
        check_product(C[b], f64(A[b]), f64(B[b]), idx[b].cpu().numpy(), product_tol(torch.bfloat16, torch.float32))
    # the stage-by-stage GEMM zeroes them with a kernel of its own
    A_S, B_S = rmm.pack(A, B, idx)
    out2 = torch.full((batch, M, N), float("nan"), device=DEV)
    C2 = rmm.gemm(A_S, B_S, idx.shape[-1], N=N, out=out2)
    assert torch.equal(C2, C)


def test_gemm_event_hook_brackets_the_gemm_kernel():
    """rmm_set_gemm_events: the events land around the GEMM kernel only (the
    split-K zeroing kernel of the stage call runs before the first one)."""
    g = torch.Generator(device=DEV)
    g.manual_seed(81)
    A_S = torch.randn(2048, 256, generator=g, device=DEV).to(torch.bfloat16)
    B_S = torch.randn(256, 1024, generator=g, device=DEV).to(torch.bfloat16)
    outer0, outer1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    C_ref = rmm.gemm(A_S, B_S, 256, N=1024)
    outer0.record()
    rmm.set_gemm_events(e0, e1)
    try:
        C = rmm.gemm(A_S, B_S, 256, N=1024)
    finally:
        rmm.set_gemm_events(None, None)
    outer1.record()
    torch.cuda.synchronize()
    assert torch.equal(C, C_ref)
    inner, outer = e0.elapsed_time(e1), outer0.elapsed_time(outer1)
    assert 0 < inner <= outer
    assert outer0.elapsed_time(e0) >= 0 and e1.elapsed_time(outer1) >= 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("b_kmajor", [False, True], ids=["rows", "kmat"])
def test_cached_b_norms(dtype, b_kmajor):
    """rmm_b_norms against the fp64 row norms of B; scores and the fused call
    with cached norms against the oracle's product-mode scores and product."""
    M, K, N = 300, 1000, 520
    A, B = _ab(M, K, N, dtype, seed=91)
    Bg = B.t().contiguous() if b_kmajor else B  # Kmat [N][K] when b_kmajor
    B64 = f64(B)
    bn = rmm.b_norms(Bg, b_kmajor=b_kmajor)
    check_scores(bn.cpu().numpy(), O.row_norms(B64))
    s = rmm.score_b_norms(A, bn)
    check_scores(s.cpu().numpy(), O.slice_scores(f64(A), B64, "product"))
    if not b_kmajor:  # B's norms are the same f32 sums as in rmm_score's product mode
        ref = rmm.score(A, B, "product")
        assert torch.allclose(s, ref, rtol=1e-6, atol=0)
    for rho in (0.3, 0.5):
        idx = torch.empty(rmm.keep_count(rho, K), dtype=torch.int32, device=DEV)
        C, ws = rmm.matmul_reduced_b_norms(A, Bg, bn, rho, idx_out=idx, b_kmajor=b_kmajor)
        rmm.check(ws)
        check_single(A, B, rho, "product", C, idx)


def test_cached_b_norms_shared_across_batch():
    """One weight for a batch of activations: b_norm [K] shared (stride 0)."""
    batch, M, K, N = 3, 256, 512, 384
    g = torch.Generator(device=DEV)
    g.manual_seed(93)
    A = torch.randn(batch, M, K, generator=g, device=DEV).to(torch.bfloat16)
    W = torch.randn(K, N, generator=g, device=DEV).to(torch.bfloat16)
    Wb = W.unsqueeze(0).expand(batch, K, N)  # batch stride 0
    bn = rmm.b_norms(W)
    idx = torch.empty(batch, rmm.keep_count(0.5, K), dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced_b_norms(A, Wb, bn, 0.5, idx_out=idx)
    rmm.check(ws)
    for b in range(batch):
        check_single(A[b], W, 0.5, "product", C[b], idx[b])


@pytest.mark.parametrize("shape,rho", [((4, 100, 128, 90), 0.3),       # k = 39: odd-length index lists, in smem
                                       ((3, 40, 40000, 24), 0.50001)],  # k = 20001 > 16384: lists read from global
                         ids=["k39", "k20001"])
def test_pack_batched_unaligned_index_lists(shape, rho):
    """Batched packs whose per-item index lists start off 16-byte boundaries
    (k_keep not a multiple of 4) take the bulk path and copy bits exactly."""
    batch, M, K, N = shape
    g = torch.Generator(device=DEV)
    g.manual_seed(97)
    A = torch.randn(batch, M, K, generator=g, device=DEV).to(torch.bfloat16)
    B = torch.randn(batch, K, N, generator=g, device=DEV).to(torch.bfloat16)
    k = rmm.keep_count(rho, K)
    assert k % 4 != 0
    s = rmm.score(A, B)
    idx = rmm.select(s, k)
    A_S, B_S = rmm.pack(A, B, idx)
    Kt = B.transpose(1, 2).contiguous()
    A_S2, Kt_S = rmm.pack(A, Kt, idx, b_kmajor=True)
    kp = rmm.padded_keep(k)
    for b in range(batch):
        I = idx[b].cpu().numpy().astype(np.int64)
        a_ref = np.zeros((M, kp)); a_ref[:, :k] = f64(A[b])[:, I]
        b_ref = np.zeros((kp, rmm.packed_b_ld(N))); b_ref[:k, :N] = f64(B[b])[I, :]
        assert np.array_equal(f64(A_S[b]), a_ref) and np.array_equal(f64(A_S2[b]), a_ref)
        assert np.array_equal(f64(B_S[b]), b_ref)
        assert np.array_equal(f64(Kt_S[b]), b_ref[:, :N].T)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 1000, 130), (3, 4096, 1000), (8, 777, 4100), (16, 2048, 257), (2, 64, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_gemv_gather_matches_oracle(shape, dtype):
    """Decode-shaped product read straight from A and B through idx: ragged
    and unaligned N, 1 to 16 rows, both output dtypes."""
    M, K, N = shape
    A, B = _ab(M, K, N, dtype, seed=M + K + N)
    A64, B64 = f64(A), f64(B)
    for rho in (0.3, 1.0):
        k = rmm.keep_count(rho, K)
        idx = rmm.select(rmm.score(A, B), k)
        for out_dtype in (torch.float32, torch.bfloat16):
            C = rmm.gemv_gather(A, B, idx, out_dtype)
            check_product(C, A64, B64, idx.cpu().numpy(), product_tol(dtype, out_dtype))
        C1 = rmm.gemv_gather(A, B, idx)
        C2 = rmm.gemv_gather(A, B, idx)
        assert torch.equal(C1, C2)  # fixed summation order


def test_gemv_gather_unaligned_rows():
    """B rows that are not 16-byte aligned (odd N, a strided view) take the
    element-wise loads."""
    M, K, N = 4, 600, 333
    A, Bfull = _ab(M, K, N + 3, torch.bfloat16, seed=5)
    B = Bfull[:, 1:N + 1]  # ld N + 3, base off by 2 bytes
    idx = rmm.select(rmm.score(A, B.contiguous()), rmm.keep_count(0.5, K))
    C = rmm.gemv_gather(A, B, idx)
    check_product(C, f64(A), f64(B), idx.cpu().numpy(), 1e-2)


@pytest.mark.parametrize("M", [1, 16])
@pytest.mark.parametrize("N,ld", [(1003, 1008), (4096, 4096)], ids=["ragged", "full"])
def test_gemv_gather_tensor_core_route(M, N, ld):
    """16-byte aligned bf16 rows take the tensor-core gather-GEMV: a ragged N
    inside an aligned row pitch (the last 16-byte copy of a row is partial),
    very few kept slices (a pass of mostly empty slots), bit-reproducible."""
    K = 3000
    A, Bfull = _ab(M, K, ld, torch.bfloat16, seed=40 + M)
    B = Bfull[:, :N]
    A64, B64 = f64(A), f64(B)
    s = rmm.score(A, B.contiguous())
    for k in (1, 33, rmm.keep_count(0.4, K)):
        idx = rmm.select(s, k)
        for out_dtype in (torch.float32, torch.bfloat16):
            C = rmm.gemv_gather(A, B, idx, out_dtype)
            check_product(C, A64, B64, idx.cpu().numpy(), product_tol(torch.bfloat16, out_dtype))
        assert torch.equal(rmm.gemv_gather(A, B, idx), rmm.gemv_gather(A, B, idx))


def test_fused_decode_shape_skips_the_pack():
    """The fused call with M <= 16 (and cached B norms, the decode setting)
    runs the selection, which computes the scores itself, and the
    gather-GEMV: 2 launches, oracle parity, one weight shared by a batch of
    sequences."""
    batch, M, K, N = 3, 4, 2048, 1536
    g = torch.Generator(device=DEV)
    g.manual_seed(101)
    X = torch.randn(batch, M, K, generator=g, device=DEV).to(torch.bfloat16)
    W = torch.randn(K, N, generator=g, device=DEV).to(torch.bfloat16)
    Wb = W.unsqueeze(0).expand(batch, K, N)
    bn = rmm.b_norms(W)
    idx = torch.empty(batch, rmm.keep_count(0.5, K), dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = rmm.launch_count()
    C, ws = rmm.matmul_reduced_b_norms(X, Wb, bn, 0.5, idx_out=idx)
    torch.cuda.synchronize()
    assert rmm.launch_count() - n0 == 2
    rmm.check(ws)
    for b in range(batch):
        check_single(X[b], W, 0.5, "product", C[b], idx[b])
    idx2 = torch.empty_like(idx)
    C2, _ = rmm.matmul_reduced(X, Wb, 0.5, idx_out=idx2)  # product score reading W, same route
    for b in range(batch):
        check_single(X[b], W, 0.5, "product", C2[b], idx2[b])


@pytest.mark.parametrize("shape", [(300, 1000, 520), (2048, 512, 1024), (256, 4096, 200), (130, 777, 1000)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fused_call_bit_identical_to_stage_calls(shape, gemm_cta_group):
    """The fused call equals, bit for bit, the stage calls pack + GEMM on its
    own kept set, for both output dtypes (ragged N, split-K last rounds whose
    C tiles the select launch zeroes, N <= 256)."""
    M, K, N = shape
    A, B = _ab(M, K, N, torch.bfloat16, seed=M + N)
    k = rmm.keep_count(0.5, K)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    for out_dtype in (torch.float32, torch.bfloat16):
        C, ws = rmm.matmul_reduced(A, B, 0.5, out_dtype=out_dtype, idx_out=idx)
        torch.cuda.synchronize()
        rmm.check(ws)
        A_S, B_S = rmm.pack(A, B, idx)
        C_ref = rmm.gemm(A_S, B_S, k, out_dtype, N=N)
        assert torch.equal(C, C_ref)
        check_product(C, f64(A), f64(B), idx.cpu().numpy(), product_tol(torch.bfloat16, out_dtype))


@pytest.mark.parametrize("K", [4096, 4097, 8192, 50000])
def test_select_large_k_with_heavy_ties(K):
    """Both compaction schemes (up to 4 keys per thread, warp sweeps beyond):
    scores drawn from 7 distinct values, so the threshold bin holds thousands
    of equal keys and only the lowest-indexed ones may be kept; batch of 3."""
    g = torch.Generator(device=DEV)
    g.manual_seed(K)
    vals = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 7.0], device=DEV)
    s = vals[torch.randint(0, 7, (3, K), generator=g, device=DEV)].contiguous()
    for rho in (0.1, 0.5, 0.93):
        k = rmm.keep_count(rho, K)
        idx = rmm.select(s, k)
        for b in range(3):
            assert idx[b].cpu().numpy().tolist() == O.select_top(s[b].cpu().numpy(), k).tolist()


@pytest.mark.parametrize("K,batch", [(2048, 1), (2049, 2), (8190, 18), (32768, 1), (32769, 1), (8192, 19)],
                         ids=lambda v: str(v))
def test_select_matches_definition_across_shapes(K, batch):
    """The selection is the definition's (largest scores, ties to the lower
    index, ascending) on the library's own f32 scores: K around the
    shared-memory limit and the compaction switch, one to 19 items, keep
    counts from 1 to K, for continuous, signed, tied and constant scores."""
    g = torch.Generator(device=DEV)
    g.manual_seed(K + batch)
    dists = {
        "lognormal": torch.exp(torch.randn(batch, K, generator=g, device=DEV)),
        "signed": torch.randn(batch, K, generator=g, device=DEV),
        "coarse": torch.randint(0, 40, (batch, K), generator=g, device=DEV).float() * 0.25,
        "constant": torch.full((batch, K), 3.0, device=DEV),
    }
    for name, s in dists.items():
        s = s.contiguous()
        for k in sorted({1, K // 2, K - 1, K}):
            idx = rmm.select(s, k)
            for b in sorted({0, batch - 1}):
                want = O.select_top(s[b].double().cpu().numpy(), k).tolist()
                assert idx[b].cpu().numpy().tolist() == want, (name, k, b)



@pytest.mark.parametrize("M,K,N,out_dtype", [(4096, 200, 4096, torch.float32), (4096, 200, 4096, torch.bfloat16),
                                              (2048, 256, 100, torch.float32), (1000, 60, 777, torch.float32)],
                         ids=["4096x200x4096-f32-split", "4096x200x4096-bf16", "2048x256x100-f32-split",
                              "1000x60x777-f32"])
def test_write_bound_gemm_epilogue(M, K, N, out_dtype):
    """Packed products with at most two k-blocks per tile (k_pad <= 128) run
    the 2-SM GEMM with 8 epilogue warps, two per TMEM lane quadrant, each
    storing half of a tile's columns; with f32 C and a partial last round
    that round is also split along K (both halves reduce-add into zeroed
    tiles; N <= 128 puts every tile there). The stage-call GEMM must match the
    oracle on rows sampled from every 256-row band (both CTAs of a pair, all
    four lane quadrants), ragged edges included, and the fused call must equal
    the stage calls of its own route bit for bit (N <= 128 streams A through
    the GEMM with B's dropped rows zeroed, a different summation order)."""
    A, B = _ab(M, K, N, torch.bfloat16, seed=M + K + N)
    k = rmm.keep_count(0.5, K)
    assert rmm.padded_keep(k) <= 128
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, B, 0.5, out_dtype=out_dtype, idx_out=idx)
    torch.cuda.synchronize()
    rmm.check(ws)
    A_S, B_S = rmm.pack(A, B, idx)
    C_packed = rmm.gemm(A_S, B_S, k, out_dtype, N=N)
    if rmm.fused_route(A, N) == rmm.ROUTE_STREAM:
        assert torch.equal(C, rmm.gemm_full(A, rmm.mask_rows(B, idx), N, out_dtype))
    else:
        assert torch.equal(C, C_packed)
    rows = sorted(set(range(0, M, 37)) | {M - 1})
    A64, B64, ii = f64(A), f64(B), idx.cpu().numpy()
    tol = product_tol(torch.bfloat16, out_dtype)
    check_product(C_packed[rows], A64[rows], B64, ii, tol)
    check_product(C[rows], A64[rows], B64, ii, tol)
