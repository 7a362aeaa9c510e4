"""GPU parity of the INT8-weight path ("Resultados Experimentais" ›
"Compatibilidade": the method works with INT8 weight quantization; read as a
per-output-column scale, W = Wq · diag(scale)) against the fp64 oracle on the
dequantized weight: row norms, the packed operand, and the fused call through
the GEMM (M > 16) and the gather-GEMV (M <= 16) routes."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O
from input_adaptive_reduced_02_b200 import inputs, rmm

from _parity import U_BF16, check_product, check_scores, check_selection, f64, product_tol

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _x(M, K, seed, batch=None):
    shape = (M, K) if batch is None else (batch, M, K)
    X, _ = inputs.outlier_activations(int(np.prod(shape[:-1])), K, 0.01, 20.0, seed, DEV)
    return X.reshape(shape).contiguous()


def _deq(Wq, scale):
    return O.dequantize_w8(Wq.cpu().numpy(), scale.cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("K,N", [(1000, 520), (777, 333), (4096, 4096)])
def test_w8_row_norms(K, N):
    Wq, scale = inputs.int8_weight(K, N, seed=K + N, device=DEV)
    bn = rmm.b_norms_w8(Wq, scale)
    check_scores(bn.cpu().numpy(), O.row_norms(_deq(Wq, scale)))


def test_w8_pack_is_the_scaled_weight_rounded_to_bf16():
    M, K, N = 200, 1000, 333
    X = _x(M, K, 1)
    Wq, scale = inputs.int8_weight(K, N, seed=2, device=DEV)
    k = rmm.keep_count(0.5, K)
    idx = rmm.select(rmm.score_b_norms(X, rmm.b_norms_w8(Wq, scale)), k)
    A_S, B_S = rmm.pack_w8(X, Wq, scale, idx)
    ii = idx.long()
    assert torch.equal(A_S[:, :k], X[:, ii]) and not A_S[:, k:].any()
    # the same f32 product, rounded to nearest even
    ref = (Wq[ii].float() * scale[None, :]).to(torch.bfloat16)
    assert torch.equal(B_S[:k, :N], ref)
    assert not B_S[k:].any() and not B_S[:, N:].any()
    # and within half a bf16 ulp (plus the f32 rounding) of the fp64 dequantized rows
    deq = _deq(Wq, scale)[idx.cpu().numpy()]
    got = f64(B_S[:k, :N])
    assert np.all(np.abs(got - deq) <= np.abs(deq) * (2.0 ** -8 + 2.0 ** -23) + 1e-30)


@pytest.mark.parametrize("M", [300, 4], ids=["gemm", "gemv"])
@pytest.mark.parametrize("mode", ["product", "a_only"])
def test_w8_fused_matches_oracle(M, mode):
    K, N = 1536, 1000
    X = _x(M, K, 3)
    Wq, scale = inputs.int8_weight(K, N, seed=4, device=DEV)
    W64 = _deq(Wq, scale)
    bn = rmm.b_norms_w8(Wq, scale) if mode == "product" else None
    for rho in (0.3, 0.5):
        k = rmm.keep_count(rho, K)
        idx = torch.empty(k, dtype=torch.int32, device=DEV)
        for out_dtype in (torch.float32, torch.bfloat16):
            C, ws = rmm.matmul_reduced_w8(X, Wq, scale, rho, b_norm=bn, mode=mode, out_dtype=out_dtype,
                                          idx_out=idx)
            rmm.check(ws)
            s_ref = O.slice_scores(f64(X), W64, mode)
            check_selection(idx.cpu().numpy(), s_ref, k)
            # the GEMM route multiplies the weight rounded to bf16; the GEMV route the exact codes
            check_product(C, f64(X), W64, idx.cpu().numpy(), product_tol(torch.bfloat16, out_dtype),
                          w_rel=U_BF16 if M > 16 else 0.0)


def test_w8_decode_batch_shares_one_weight():
    batch, M, K, N = 3, 2, 2048, 1100
    X = _x(M, K, 5, batch=batch)
    Wq, scale = inputs.int8_weight(K, N, seed=6, device=DEV)
    Wb = Wq.unsqueeze(0).expand(batch, K, N)
    bn = rmm.b_norms_w8(Wq, scale)
    idx = torch.empty(batch, rmm.keep_count(0.5, K), dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced_w8(X, Wb, scale, 0.5, b_norm=bn, idx_out=idx)
    rmm.check(ws)
    W64 = _deq(Wq, scale)
    for b in range(batch):
        check_selection(idx[b].cpu().numpy(), O.slice_scores(f64(X[b]), W64), idx.shape[1])
        check_product(C[b], f64(X[b]), W64, idx[b].cpu().numpy(), 1e-2)


def test_w8_rejects_misaligned_weights_and_missing_norms():
    X = _x(8, 64, 7)
    Wq, scale = inputs.int8_weight(64, 40, seed=8, device=DEV)
    with pytest.raises(ValueError):
        rmm.matmul_reduced_w8(X, Wq, scale, 0.5)  # product mode without b_norm
    Wodd = torch.zeros(64, 43, dtype=torch.int8, device=DEV)[:, 1:41]  # rows 43 bytes apart
    rmm.b_norms_w8(Wodd, scale)  # any alignment
    with pytest.raises(rmm.RMMError) as e:  # the gather-GEMV copies 4 int8 at a time
        rmm.matmul_reduced_w8(X, Wodd, scale, 0.5, mode="a_only")
    assert e.value.status == rmm.RMM_ERR_UNSUPPORTED


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("N,ld", [(1000, 1024), (4096, 4096)], ids=["ragged", "full"])
def test_w8_gemv_tensor_core_route(M, N, ld):
    """16-byte aligned INT8 rows take the tensor-core gather-GEMV (int8 rows
    converted exactly to bf16 per pass); a ragged N inside a wider row pitch
    checks the column bounds."""
    K = 3000
    X = _x(M, K, 11 + M)
    Wfull, sfull = inputs.int8_weight(K, ld, seed=12, device=DEV)
    Wq, scale = Wfull[:, :N], sfull[:N].contiguous()
    W64 = _deq(Wq, scale)
    bn = rmm.b_norms_w8(Wq, scale)
    k = rmm.keep_count(0.4, K)
    idx = rmm.select(rmm.score_b_norms(X, bn), k)
    for out_dtype in (torch.float32, torch.bfloat16):
        C = rmm.gemv_gather_w8(X, Wq, scale, idx, out_dtype)
        check_product(C, f64(X), W64, idx.cpu().numpy(), product_tol(torch.bfloat16, out_dtype))
    assert torch.equal(rmm.gemv_gather_w8(X, Wq, scale, idx), rmm.gemv_gather_w8(X, Wq, scale, idx))
    for k_small in (1, 33):  # a pass of mostly empty slots
        idx_s = rmm.select(rmm.score_b_norms(X, bn), k_small)
        C = rmm.gemv_gather_w8(X, Wq, scale, idx_s)
        check_product(C, f64(X), W64, idx_s.cpu().numpy(), product_tol(torch.bfloat16, torch.float32))
