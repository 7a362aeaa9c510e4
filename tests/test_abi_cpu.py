"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/rmm.h declares, and its host helpers and argument
validation behave as documented (validation runs before any CUDA call)."""
from __future__ import annotations

import ctypes
import math
import os
import re
from fractions import Fraction

import pytest

from input_adaptive_reduced_02_b200 import rmm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rmm.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(rmm_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_library_loads_and_exports_every_declared_symbol():
    L = rmm.lib()
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), f"{n} declared in rmm.h but not exported"
    assert set(names) == set(rmm._SIGS), "binding signatures out of sync with rmm.h"


def test_keep_count_matches_exact_ceiling():
    for K in [1, 2, 3, 7, 10, 64, 128, 256, 1000, 4096, 8192, 16384, 28672, 32768]:
        for rho in [0.01, 0.1, 0.25, 0.3, 0.5, 0.7, 0.9, 1.0]:
            assert rmm.keep_count(rho, K) == max(1, math.ceil(Fraction(str(rho)) * K)), (rho, K)
    L = rmm.lib()
    for bad in (0.0, -1.0, 1.5, float("nan"), float("inf")):
        assert L.rmm_keep_count(bad, 10) == -1
    assert L.rmm_keep_count(0.5, 0) == -1
    assert L.rmm_keep_count(1e-300, 10) == 1


def test_padded_keep_and_workspace_layout():
    assert rmm.padded_keep(1) == 64 and rmm.padded_keep(64) == 64 and rmm.padded_keep(65) == 128
    ws = rmm.workspace_size(1, 4096, 4096, 4096, 2048, rmm.torch.bfloat16)
    # status + scores + indices + A_S + packed B, each 1 KiB aligned
    expect = 1024 + 4096 * 4 + 2048 * 4 + 4096 * 2048 * 2 + 4096 * 2048 * 2
    assert ws == expect
    ws32 = rmm.workspace_size(2, 3, 5, 7, 3, rmm.torch.float32)
    # A_S: 2*3*64*4 = 1536 -> 2048; packed B: 2*64*8*4 = 4096 (row pitch 7 -> 8)
    assert ws32 == 1024 + 1024 + 1024 + 2048 + 4096


def test_workspace_size_for_the_decode_route():
    """With M <= 16 and B row-major the fused calls pack nothing: the workspace
    they need is the status word, scores and indices; other routes need the
    packed operands too."""
    al = lambda x: (x + 1023) // 1024 * 1024  # noqa: E731
    K, N, k = 8192, 28672, 4096
    decode = rmm.workspace_size_for(1, 1, K, N, k, rmm.torch.bfloat16)
    assert decode == al(4) + al(K * 4) + al(k * 4) == 50176
    full = rmm.workspace_size(1, 1, K, N, k, rmm.torch.bfloat16)
    assert full > 200 * 2**20 and decode < full
    assert rmm.workspace_size_for(1, 1, K, N, k, rmm.torch.bfloat16, b_kmajor=True) == full
    assert rmm.workspace_size_for(1, 17, K, N, k, rmm.torch.bfloat16) == rmm.workspace_size(1, 17, K, N, k,
                                                                                               rmm.torch.bfloat16)
    assert rmm.workspace_size_for(3, 16, K, N, k, rmm.torch.float32) == al(4) + al(3 * K * 4) + al(3 * k * 4)


def test_workspace_size_for_the_stream_route():
    """bf16, B row-major, N <= 128, M > 16 (P·V): the fused calls stream A whole
    and need B with its dropped rows zeroed, [batch][K][packed_b_ld(N)],
    instead of the packed operands; rmm_workspace_size covers both routes."""
    al = lambda x: (x + 1023) // 1024 * 1024  # noqa: E731
    bh, S, d, rho = 32, 32768, 128, 0.5
    k = rmm.keep_count(rho, S)
    stream = rmm.workspace_size_for(bh, S, S, d, k, rmm.torch.bfloat16)
    head = al(4) + al(bh * S * 4) + al(bh * k * 4)
    assert stream == head + al(bh * S * d * 2)
    pack = head + al(bh * S * k * 2) + al(bh * k * d * 2)
    assert rmm.workspace_size(bh, S, S, d, k, rmm.torch.bfloat16) == max(pack, stream) == pack
    assert stream < pack / 100
    # f32, a K-major B or N > 128 take the pack route
    assert rmm.workspace_size_for(bh, S, S, d, k, rmm.torch.bfloat16, b_kmajor=True) == pack
    assert rmm.workspace_size_for(1, 300, 1000, 129, 500, rmm.torch.bfloat16) == \
        rmm.workspace_size(1, 300, 1000, 129, 500, rmm.torch.bfloat16)
    # few rows of A and a wide K: the stream operand is the larger one
    M, K, N, k = 17, 8192, 128, 4096
    s2 = rmm.workspace_size_for(1, M, K, N, k, rmm.torch.bfloat16)
    assert s2 == al(4) + al(K * 4) + al(k * 4) + al(K * N * 2)
    assert rmm.workspace_size(1, M, K, N, k, rmm.torch.bfloat16) == s2


def test_fused_route_rule():
    """rmm_fused_route: the gather-GEMV for M <= 16 with B row-major, the stream
    route for narrow bf16 products whose A can be streamed, the pack route
    otherwise; it only inspects the pointer's alignment."""
    L = rmm.lib()
    a = V(1 << 20)
    assert L.rmm_fused_route(1, 16, 4096, 0, 0, a, 4096, 0) == 2
    assert L.rmm_fused_route(32, 8192, 128, 0, 0, a, 8192, 8192 * 8192) == 1
    assert L.rmm_fused_route(32, 8192, 128, 0, 1, a, 8192, 8192 * 8192) == 0   # f32
    assert L.rmm_fused_route(32, 8192, 128, 1, 0, a, 8192, 8192 * 8192) == 0   # K-major B
    assert L.rmm_fused_route(32, 8192, 129, 0, 0, a, 8192, 8192 * 8192) == 0   # wider than one tile
    assert L.rmm_fused_route(1, 700, 128, 0, 0, a, 700, 0) == 0                # row pitch not 16 bytes
    assert L.rmm_fused_route(1, 700, 128, 0, 0, V((1 << 20) + 2), 704, 0) == 0  # base not 16-byte aligned
    assert L.rmm_fused_route(2, 700, 128, 0, 0, a, 704, 0) == 0                # one A shared by the batch
    assert L.rmm_fused_route(-1, 700, 128, 0, 0, a, 704, 0) == -1


V = ctypes.c_void_p


def test_fused_calls_accept_the_route_workspace():
    """The fused call's workspace check follows its route: a decode-shaped call
    (M = 4, B row-major) passes it with exactly rmm_workspace_size_for bytes and
    fails it with one byte less; a K-major B needs the full size."""
    L = rmm.lib()
    null = V(0)
    M, K, N = 4, 64, 40
    k = rmm.keep_count(0.5, K)
    need = rmm.workspace_size_for(1, M, K, N, k, rmm.torch.bfloat16)
    # rmm_matmul_reduced_batched(A, lda, sA, B, ldb, sB, b_kmajor, batch, M, K, N, rho, in, mode, C, ldc, sC, out,
    #                            idx_out, workspace, bytes, stream)
    def call(b_kmajor, ldb, nbytes):
        return L.rmm_matmul_reduced_batched(V(1 << 20), K, 0, V(1 << 20), ldb, 0, b_kmajor, 1, M, K, N, 0.5, 0, 0,
                                            V(1 << 20), N, 0, 1, null, V(1 << 30), nbytes, null)
    assert call(0, N, need - 1) == rmm.RMM_ERR_INVALID
    assert b"workspace too small" in L.rmm_last_error_string()
    assert call(1, K, need) == rmm.RMM_ERR_INVALID  # K-major B: the pack route needs the packed operands
    assert b"workspace too small" in L.rmm_last_error_string()
    if not rmm.torch.cuda.is_available():
        # Past the workspace check the call goes on to bind a device, which
        # fails without a GPU. (With a GPU these pointers would reach kernels,
        # so the accepting half runs only where there is none.)
        full = rmm.workspace_size(1, M, K, N, k, rmm.torch.bfloat16)
        assert call(0, N, need) == rmm.RMM_ERR_CUDA
        assert call(1, K, full) == rmm.RMM_ERR_CUDA


def test_validation_errors_need_no_gpu():
    L = rmm.lib()
    null = V(0)
    # rho outside (0, 1]
    st = L.rmm_matmul_reduced(V(16), 8, V(16), 8, 4, 8, 8, 1.5, 0, 0, V(16), 8, 1, null, V(1024), 1 << 20, null)
    assert st == rmm.RMM_ERR_INVALID
    assert b"rho" in L.rmm_last_error_string()
    # A is NULL
    st = L.rmm_matmul_reduced(null, 8, V(16), 8, 4, 8, 8, 0.5, 0, 0, V(16), 8, 1, null, V(1024), 1 << 20, null)
    assert st == rmm.RMM_ERR_INVALID
    # leading dimension smaller than the row
    st = L.rmm_score(V(16), 4, 0, V(16), 8, 0, 0, 1, 4, 8, 8, 0, 0, V(16), null, null)
    assert st == rmm.RMM_ERR_INVALID
    # workspace too small
    st = L.rmm_matmul_reduced(V(16), 8, V(16), 8, 4, 8, 8, 0.5, 0, 0, V(16), 8, 1, null, V(1024), 16, null)
    assert st == rmm.RMM_ERR_INVALID and b"workspace" in L.rmm_last_error_string()
    # misaligned workspace
    st = L.rmm_matmul_reduced(V(16), 8, V(16), 8, 4, 8, 8, 0.5, 0, 0, V(16), 8, 1, null, V(1040), 1 << 20, null)
    assert st == rmm.RMM_ERR_INVALID
    # k_keep outside [1, K]
    assert L.rmm_select(V(16), 1, 10, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_select(V(16), 1, 10, 11, V(16), null, null) == rmm.RMM_ERR_INVALID
    # unknown dtype / score mode
    assert L.rmm_score(V(16), 8, 0, V(16), 8, 0, 0, 1, 4, 8, 8, 7, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_score(V(16), 8, 0, V(16), 8, 0, 0, 1, 4, 8, 8, 0, 9, V(16), null, null) == rmm.RMM_ERR_INVALID
    # K = 0
    assert L.rmm_score(V(16), 8, 0, V(16), 8, 0, 0, 1, 4, 0, 8, 0, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    # empty batch is a no-op that needs no device
    assert L.rmm_select(null, 0, 10, 3, null, null, null) == rmm.RMM_OK


def test_cached_b_norm_calls_validate_without_gpu():
    L = rmm.lib()
    null = V(0)
    # rmm_b_norms: B or the output missing; ld smaller than a row
    assert L.rmm_b_norms(null, 8, 0, 0, 1, 8, 8, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_b_norms(V(16), 8, 0, 0, 1, 8, 8, 0, null, null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_b_norms(V(16), 4, 0, 0, 1, 8, 8, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    # rmm_score_b_norms: norms missing; a batch stride between 0 and K
    assert L.rmm_score_b_norms(V(16), 8, 64, null, 0, 2, 4, 8, 0, V(16), null, null) == rmm.RMM_ERR_INVALID
    st = L.rmm_score_b_norms(V(16), 8, 64, V(16), 3, 2, 4, 8, 0, V(16), null, null)
    assert st == rmm.RMM_ERR_INVALID and b"b_norm_stride" in L.rmm_last_error_string()
    # fused: rho outside (0, 1] is still caught
    st = L.rmm_matmul_reduced_b_norms(V(16), 8, 0, V(16), 8, 0, 0, V(16), 0, 1, 4, 8, 8, 0.0, 0, V(16), 8, 0, 1,
                                      null, V(1024), 1 << 20, null)
    assert st == rmm.RMM_ERR_INVALID and b"rho" in L.rmm_last_error_string()


def test_gemv_and_int8_calls_validate_without_gpu():
    L = rmm.lib()
    null = V(0)
    BF16, F32 = 0, 1
    # rmm_gemv_gather(A, lda, sA, B, ldb, sB, batch, M, K, N, idx, k_keep, in, C, ldc, sC, out, stream)
    gv = [V(16), 8, 0, V(16), 8, 0, 1, 4, 8, 8, V(16), 3, BF16, V(16), 8, 0, F32, null]

    def with_(args, pos, value):
        a = list(args)
        a[pos] = value
        return a

    assert L.rmm_gemv_gather(*with_(gv, 7, 17)) == rmm.RMM_ERR_INVALID  # M above 16
    assert b"16" in L.rmm_last_error_string()
    assert L.rmm_gemv_gather(*with_(gv, 11, 0)) == rmm.RMM_ERR_INVALID  # k_keep outside [1, K]
    assert L.rmm_gemv_gather(*with_(gv, 11, 9)) == rmm.RMM_ERR_INVALID
    assert L.rmm_gemv_gather(*with_(gv, 10, null)) == rmm.RMM_ERR_INVALID  # idx missing
    assert L.rmm_gemv_gather(*with_(gv, 14, 4)) == rmm.RMM_ERR_INVALID  # ldc smaller than N
    assert L.rmm_gemv_gather(*with_(gv, 16, 7)) == rmm.RMM_ERR_INVALID  # unknown output dtype
    assert L.rmm_gemv_gather(*with_(gv, 6, 0)) == rmm.RMM_OK  # empty batch: nothing to do, no device needed
    # rmm_b_norms_w8(Wq, ldw, sW, scale, ss, batch, K, N, out, status, stream)
    assert L.rmm_b_norms_w8(null, 8, 0, V(16), 0, 1, 8, 8, V(16), null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_b_norms_w8(V(16), 8, 0, null, 0, 1, 8, 8, V(16), null, null) == rmm.RMM_ERR_INVALID
    assert L.rmm_b_norms_w8(V(16), 4, 0, V(16), 0, 1, 8, 8, V(16), null, null) == rmm.RMM_ERR_INVALID
    # a per-item scale stride that would overlap the items' scales
    assert L.rmm_b_norms_w8(V(16), 8, 64, V(16), 3, 2, 8, 8, V(16), null, null) == rmm.RMM_ERR_INVALID
    # rmm_gemv_gather_w8(A, lda, sA, Wq, ldw, sW, scale, ss, batch, M, K, N, idx, k, C, ldc, sC, out, stream)
    w8 = [V(16), 8, 0, V(16), 8, 0, V(16), 0, 1, 4, 8, 8, V(16), 3, V(16), 8, 0, F32, null]
    assert L.rmm_gemv_gather_w8(*with_(w8, 9, 17)) == rmm.RMM_ERR_INVALID  # M above 16
    # int8 rows not 4-byte aligned (base, then row pitch)
    assert L.rmm_gemv_gather_w8(*with_(w8, 3, V(17))) == rmm.RMM_ERR_UNSUPPORTED
    assert L.rmm_gemv_gather_w8(*with_(w8, 4, 10)) == rmm.RMM_ERR_UNSUPPORTED
    # rmm_matmul_reduced_w8(A, lda, sA, Wq, ldw, sW, scale, ss, b_norm, bns, batch, M, K, N, rho, in, mode,
    #                       C, ldc, sC, out, idx_out, workspace, ws_bytes, stream)
    f = [V(16), 8, 0, V(16), 8, 0, V(16), 0, V(16), 0, 1, 4, 8, 8, 0.5, BF16, 0, V(16), 8, 0, F32, null,
         V(1024), 1 << 20, null]
    assert L.rmm_matmul_reduced_w8(*with_(f, 15, F32)) == rmm.RMM_ERR_INVALID  # activations must be bf16
    assert L.rmm_matmul_reduced_w8(*with_(f, 8, null)) == rmm.RMM_ERR_INVALID  # product score needs W's norms
    assert L.rmm_matmul_reduced_w8(*with_(f, 16, 5)) == rmm.RMM_ERR_INVALID  # unknown score mode
    assert L.rmm_matmul_reduced_w8(*with_(f, 14, 0.0)) == rmm.RMM_ERR_INVALID  # rho outside (0, 1]
    assert L.rmm_matmul_reduced_w8(*with_(f, 23, 16)) == rmm.RMM_ERR_INVALID  # workspace too small
    # rmm_pack_w8(A, lda, sA, Wq, ldw, sW, scale, ss, batch, M, K, N, idx, k, A_S, B_S, status, stream)
    pk = [V(16), 8, 0, V(16), 8, 0, V(16), 0, 1, 4, 8, 8, V(16), 3, V(16), V(16), null, null]
    assert L.rmm_pack_w8(*with_(pk, 12, null)) == rmm.RMM_ERR_INVALID  # idx missing
    assert L.rmm_pack_w8(*with_(pk, 13, 9)) == rmm.RMM_ERR_INVALID  # k_keep above K


def test_binding_refuses_cpu_tensors():
    A = rmm.torch.zeros(4, 8, dtype=rmm.torch.bfloat16)
    with pytest.raises(ValueError):
        rmm.score(A, A.t().contiguous())
