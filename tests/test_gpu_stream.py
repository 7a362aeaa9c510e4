"""The stream route ("Mecanismo Central": A[:, I]·B[I, :] = A·B_M with B_M the
rows of B in I and zeros elsewhere): rmm_mask_rows bit for bit against its
definition, rmm_gemm_full and the fused calls that take this route (bf16,
B row-major, N <= 128, M > 16: P·V) against the fp64 oracle's product over
the kept set, ragged K and N, batches, one kept slice and all of them."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O
from input_adaptive_reduced_02_b200 import inputs, rmm

from _parity import check_product, check_single, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _ab(batch, M, K, N, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    A = torch.randn(batch, M, K, generator=g, device=DEV) * torch.exp(torch.randn(batch, 1, K, generator=g, device=DEV))
    B = torch.randn(batch, K, N, generator=g, device=DEV)
    return A.to(dtype).contiguous(), B.to(dtype).contiguous()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 1000, 100), (3, 777, 128), (2, 64, 1), (1, 4096, 37)],
                         ids=lambda s: "x".join(map(str, s)))
def test_mask_rows_is_the_definition(shape, dtype):
    batch, K, N = shape
    g = torch.Generator(device=DEV)
    g.manual_seed(K + N)
    B = torch.randn(batch, K, N, generator=g, device=DEV).to(dtype)
    s = torch.rand(batch, K, generator=g, device=DEV)
    ldm = rmm.packed_b_ld(N)
    for k in sorted({1, K // 3, K - 1, K} - {0}):
        idx = rmm.select(s, k)
        Bm = rmm.mask_rows(B, idx)
        assert Bm.shape == (batch, K, ldm)
        for b in range(batch):
            want = torch.zeros(K, ldm, dtype=dtype, device=DEV)
            ii = idx[b].long()
            want[ii, :N] = B[b][ii]
            assert torch.equal(Bm[b], want), (k, b)


@pytest.mark.parametrize("shape", [(1, 300, 1000, 100), (3, 129, 64, 128), (2, 1000, 2056, 1), (1, 17, 4096, 128)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32out", "bf16out"])
def test_gemm_full_is_the_reduced_product(shape, out_dtype):
    batch, M, K, N = shape
    A, B = _ab(batch, M, K, N, torch.bfloat16, seed=M + K)
    s = rmm.score(A, B)
    for rho in (0.3, 1.0):
        k = rmm.keep_count(rho, K)
        idx = rmm.select(s, k)
        C = rmm.gemm_full(A, rmm.mask_rows(B, idx), N, out_dtype)
        for b in range(batch):
            check_product(C[b], f64(A[b]), f64(B[b]), idx[b].cpu().numpy(), 1e-2)


@pytest.mark.parametrize("shape", [(1, 300, 1000, 100), (4, 200, 512, 128), (1, 17, 2048, 64)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("rho", [1e-9, 0.3, 0.5, 1.0])
def test_fused_call_takes_the_stream_route(shape, rho):
    batch, M, K, N = shape
    A, B = _ab(batch, M, K, N, torch.bfloat16, seed=3 * M + N)
    assert rmm.fused_route(A, N) == rmm.ROUTE_STREAM
    k = rmm.keep_count(rho, K)
    idx = torch.empty(batch, k, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = rmm.launch_count()
    C, ws = rmm.matmul_reduced(A, B, rho, idx_out=idx)
    torch.cuda.synchronize()
    assert rmm.launch_count() - n0 == 4  # score, select, mask, gemm
    assert ws.nbytes == rmm.workspace_size_for(batch, M, K, N, k, torch.bfloat16)
    rmm.check(ws)
    for b in range(batch):
        check_single(A[b], B[b], rho, "product", C[b], idx[b])
    # the same kernels as the stage calls, bit for bit
    C2 = rmm.gemm_full(A, rmm.mask_rows(B, idx), N)
    assert torch.equal(C, C2)


@pytest.mark.parametrize("S", [1000, 2048])
def test_pv_reduced_stream_route(S):
    P, V = inputs.attention_pv(bh=3, S=S, d=128, seed=5, device=DEV)
    assert rmm.fused_route(P, 128) == rmm.ROUTE_STREAM
    for rho in (0.3, 0.5, 0.7):
        k = rmm.keep_count(rho, S)
        idx = torch.empty(3, k, dtype=torch.int32, device=DEV)
        Oo, ws = rmm.pv_reduced(P, V, rho, idx_out=idx)
        rmm.check(ws)
        for h in range(3):
            check_single(P[h], V[h], rho, "product", Oo[h], idx[h])


def test_unaligned_a_falls_back_to_the_pack_route():
    """A row pitch that is not a multiple of 8 elements cannot be streamed by
    TMA: the call packs, with the larger workspace, and gives the same
    product up to f32 rounding order."""
    A0, B = _ab(1, 200, 1001, 100, torch.bfloat16, seed=9)
    A = A0[0][:, :1000]  # row pitch 1001
    Bm = B[0][:1000].contiguous()
    assert rmm.fused_route(A, 100) == rmm.ROUTE_PACK
    idx = torch.empty(rmm.keep_count(0.5, 1000), dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced(A, Bm, 0.5, idx_out=idx)
    assert ws.nbytes == rmm.workspace_size(1, 200, 1000, 100, idx.numel(), torch.bfloat16)
    rmm.check(ws)
    check_single(A.contiguous(), Bm, 0.5, "product", C, idx)
    Ac = A.contiguous()
    assert rmm.fused_route(Ac, 100) == rmm.ROUTE_STREAM
    C2, _ = rmm.matmul_reduced(Ac, Bm, 0.5)
    assert O.frobenius_rel_error(f64(C2), f64(C)) < 1e-5
