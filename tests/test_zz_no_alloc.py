"""rmm_matmul_reduced_noalloc: the allocation-free entry point, for callers
that must not allocate device memory (for example code running under another
framework's allocator, or a plugin handed only its input and output buffers).
Its scratch is the library's static 32 MiB device array. Called here through
the C ABI and compared with rmm_matmul_reduced (workspace form) on two calls
in a row, so the second call runs on scratch the first one left behind:
bit-identical output and indices, and the fp64 oracle's selection and
product."""
from __future__ import annotations

import ctypes

import pytest
import torch

from input_adaptive_reduced_02_b200 import rmm

from _parity import check_single

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    A = torch.randn(M, K, generator=g, device="cuda") * torch.exp(torch.randn(K, generator=g, device="cuda"))
    B = torch.randn(K, N, generator=g, device="cuda")
    return A.to(torch.bfloat16).contiguous(), B.to(torch.bfloat16).contiguous()


def _call_noalloc(A, B, rho, C, idx, status):
    L = rmm.lib()
    M, K = A.shape
    N = B.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.rmm_matmul_reduced_noalloc(
        ctypes.c_void_p(A.data_ptr()), A.stride(0), ctypes.c_void_p(B.data_ptr()), B.stride(0), M, K, N,
        float(rho), rmm.RMM_BF16, 0, ctypes.c_void_p(C.data_ptr()), C.stride(0), rmm.RMM_F32,
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(status.data_ptr()), stream)


@pytest.mark.parametrize("first,second", [((384, 1536, 640, 0.5, 1), (300, 1000, 520, 0.3, 2))])
def test_noalloc_matches_workspace_entry_point_on_two_calls(first, second):
    for M, K, N, rho, seed in (first, second):
        A, B = _inputs(M, K, N, seed)
        k = rmm.keep_count(rho, K)
        idx_ref = torch.empty(k, dtype=torch.int32, device="cuda")
        C_ref, ws = rmm.matmul_reduced(A, B, rho, idx_out=idx_ref)
        rmm.check(ws)

        C = torch.full((M, N), float("nan"), device="cuda")
        idx = torch.full((k,), -1, dtype=torch.int32, device="cuda")
        status = rmm.status_word()
        assert _call_noalloc(A, B, rho, C, idx, status) == rmm.RMM_OK, rmm.lib().rmm_last_error_string()
        rmm.check(status)
        torch.cuda.synchronize()
        # same route, same kernels: identical bits, whatever the first call left in the scratch
        assert torch.equal(idx, idx_ref)
        assert torch.equal(C, C_ref)
        # and the fp64 oracle's selection and product over the kept slices
        check_single(A, B, rho, "product", C, idx)


def test_noalloc_rejects_products_beyond_its_scratch():
    A, B = _inputs(4096, 4096, 4096, 3)  # needs ~32 MiB of packed operands plus scores at rho = 0.5
    C = torch.empty(4096, 4096, device="cuda")
    idx = torch.empty(rmm.keep_count(0.5, 4096), dtype=torch.int32, device="cuda")
    st = _call_noalloc(A, B, 0.5, C, idx, rmm.status_word())
    assert st == rmm.RMM_ERR_INVALID
    assert b"static scratch" in rmm.lib().rmm_last_error_string()


def test_noalloc_takes_decode_products_beyond_its_scratch():
    """A decode-shaped product (one row of A, B row-major) packs nothing, so its
    scratch is scores and indices only: a weight whose packed rows alone would
    take 64 MiB runs through the static 32 MiB scratch, bit-identical to the
    workspace entry point (same route, same kernels)."""
    M, K, N, rho = 1, 4096, 16384, 0.5
    k = rmm.keep_count(rho, K)
    assert rmm.workspace_size(1, M, K, N, k, torch.bfloat16) > 32 * 2**20
    A, B = _inputs(M, K, N, 4)
    idx_ref = torch.empty(k, dtype=torch.int32, device="cuda")
    C_ref, ws = rmm.matmul_reduced(A, B, rho, idx_out=idx_ref)
    assert ws.nbytes == rmm.workspace_size_for(1, M, K, N, k, torch.bfloat16)
    rmm.check(ws)
    C = torch.full((M, N), float("nan"), device="cuda")
    idx = torch.full((k,), -1, dtype=torch.int32, device="cuda")
    status = rmm.status_word()
    assert _call_noalloc(A, B, rho, C, idx, status) == rmm.RMM_OK, rmm.lib().rmm_last_error_string()
    rmm.check(status)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_ref)
    assert torch.equal(C, C_ref)

