"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (the fused calls). Where the fp64 oracle cannot afford the
whole product, it is applied to sub-problems whose answers the full result
must contain exactly: a product entry depends only on its row of A and its
column of B, and a slice score only on column k of A and row k of B.
The integer stage (selection) is always checked on every head/matrix:
bit-exact against the oracle's selection on the library's f32 scores, with
the scores themselves checked against fp64."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O
from input_adaptive_reduced_02_b200 import inputs, rmm

from _parity import U_BF16, check_index_list, check_product, check_scores, check_selection, f64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

DEV = "cuda"


def _rows_cols(M, N, nr, nc, seed):
    r = np.random.default_rng(seed)
    rows = np.sort(r.choice(M, size=min(nr, M), replace=False))
    cols = np.sort(r.choice(N, size=min(nc, N), replace=False))
    return rows, cols


def _check_selection_exact(s_gpu: torch.Tensor, idx_gpu: torch.Tensor, k: int):
    check_index_list(idx_gpu.cpu().numpy(), s_gpu.shape[-1], k)
    assert idx_gpu.cpu().numpy().tolist() == O.select_top(s_gpu.cpu().numpy(), k).tolist()


def test_linear_4096_all_rhos_full_compare():
    X, W = inputs.linear_projection(seed=0, device=DEV)
    X64, W64 = f64(X), f64(W)
    s_ref = O.slice_scores(X64, W64)
    s = rmm.score(X, W)
    check_scores(s.cpu().numpy(), s_ref)
    ws = None
    for rho in (0.3, 0.5, 0.7, 0.9, 1.0):
        k = rmm.keep_count(rho, 4096)
        idx = torch.empty(k, dtype=torch.int32, device=DEV)
        C, ws = rmm.matmul_reduced(X, W, rho, idx_out=idx, workspace=ws)
        rmm.check(ws)
        _check_selection_exact(s, idx, k)
        check_selection(idx.cpu().numpy(), s_ref, k)
        check_product(C, X64, W64, idx.cpu().numpy(), 1e-2)


def test_qk_32x4096x128():
    Q, Km = inputs.attention_qk(seed=0, device=DEV)
    k = rmm.keep_count(0.5, 128)
    idx = torch.empty(32, k, dtype=torch.int32, device=DEV)
    S, ws = rmm.qk_reduced(Q, Km, 0.5, out_dtype=torch.float32, idx_out=idx)
    rmm.check(ws)
    s = rmm.score(Q, Km, b_kmajor=True)
    for h in range(32):
        Q64, K64 = f64(Q[h]), f64(Km[h])
        s_ref = O.slice_scores(Q64, K64.T)
        check_scores(s[h].cpu().numpy(), s_ref)
        _check_selection_exact(s[h], idx[h], k)
        check_selection(idx[h].cpu().numpy(), s_ref, k)
        rows, cols = _rows_cols(4096, 4096, 128, 512, h)
        check_product(S[h][rows][:, cols], Q64[rows], K64[cols].T, idx[h].cpu().numpy(), 1e-2)
    # two heads in full
    for h in (0, 31):
        check_product(S[h], f64(Q[h]), f64(Km[h]).T, idx[h].cpu().numpy(), 1e-2)


@pytest.mark.parametrize("S", [8192, 16384, 32768])
def test_pv_long_context(S):
    heads_checked = [0, 17]
    P, V = inputs.attention_pv(bh=32, S=S, d=128, seed=0, device=DEV)
    ws = None
    s = rmm.score(P, V)
    for rho in (0.3, 0.5, 0.7):
        k = rmm.keep_count(rho, S)
        idx = torch.empty(32, k, dtype=torch.int32, device=DEV)
        Oo, ws = rmm.pv_reduced(P, V, rho, idx_out=idx, workspace=ws)
        rmm.check(ws)
        for h in range(32):
            _check_selection_exact(s[h], idx[h], k)
        for h in heads_checked:
            rows, cols = _rows_cols(S, S, 256, 1024, h + S)
            # scores of sampled slices against fp64
            P_cols = f64(P[h][:, torch.as_tensor(cols, device=DEV)])
            s_ref_cols = O.slice_scores(P_cols, f64(V[h][torch.as_tensor(cols, device=DEV)]))
            check_scores(s[h][torch.as_tensor(cols, device=DEV)].cpu().numpy(), s_ref_cols)
            # sampled output rows: O[r, :] = P[r, I] · V[I, :], whole rows of P
            rr = torch.as_tensor(rows, device=DEV)
            check_product(Oo[h][rr], f64(P[h][rr]), f64(V[h]), idx[h].cpu().numpy(), 1e-2)
    del P, V, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("which", ["up", "down"])
def test_mlp_70b_projections(which):
    X, W = (inputs.mlp_up if which == "up" else inputs.mlp_down)(seed=0, device=DEV)
    M, K = X.shape
    N = W.shape[1]
    s = rmm.score(X, W)
    # all scores in fp64, column by column block to bound host memory
    s_ref = np.concatenate([O.slice_scores(f64(X[:, c0:c0 + 4096]), f64(W[c0:c0 + 4096]))
                            for c0 in range(0, K, 4096)])
    check_scores(s.cpu().numpy(), s_ref)
    ws = None
    for rho in (0.5, 0.7, 0.9):
        k = rmm.keep_count(rho, K)
        idx = torch.empty(k, dtype=torch.int32, device=DEV)
        C, ws = rmm.matmul_reduced(X, W, rho, idx_out=idx, workspace=ws)
        rmm.check(ws)
        _check_selection_exact(s, idx, k)
        check_selection(idx.cpu().numpy(), s_ref, k)
        rows, cols = _rows_cols(M, N, 128, 512, k)
        ii = idx.long()
        A_sub = f64(X[torch.as_tensor(rows, device=DEV)])
        B_sub = f64(W[:, torch.as_tensor(cols, device=DEV)])
        check_product(C[torch.as_tensor(rows, device=DEV)][:, torch.as_tensor(cols, device=DEV)],
                      A_sub, B_sub, idx.cpu().numpy(), 1e-2)
    del X, W, ws
    torch.cuda.empty_cache()


def _block_scores(X: torch.Tensor, W64_rows, K: int, rows: int = 1024) -> np.ndarray:
    """fp64 slice scores of x · W, 1024 slices at a time (slice k needs only
    column k of x and row k of W); W64_rows(r0, r1) gives W[r0:r1] in fp64."""
    return np.concatenate([O.slice_scores(f64(X[:, r0:r0 + rows]), W64_rows(r0, min(K, r0 + rows)))
                           for r0 in range(0, K, rows)])


@pytest.mark.parametrize("M", [1, 16])
def test_decode_mlp_up_full_size(M):
    """Decode on the full MLP-up weight, x[M×8192] · W[8192×28672] with W's
    norms cached, through the fused call the benchmark times: every score
    against fp64, the selection bit-exact on the library's scores and within
    the near-tie rule against fp64, the product on 1024 sampled columns."""
    X, W = inputs.mlp_up(seed=0, device=DEV)
    X = X[:M].contiguous()
    K, N = W.shape
    bn = rmm.b_norms(W)
    s = rmm.score_b_norms(X, bn)
    s_ref = _block_scores(X, lambda r0, r1: f64(W[r0:r1]), K)
    check_scores(s.cpu().numpy(), s_ref)
    for rho in (0.5, 0.3):
        k = rmm.keep_count(rho, K)
        idx = torch.empty(k, dtype=torch.int32, device=DEV)
        C, ws = rmm.matmul_reduced_b_norms(X, W, bn, rho, idx_out=idx)
        rmm.check(ws)
        _check_selection_exact(s, idx, k)
        check_selection(idx.cpu().numpy(), s_ref, k)
        _, cols = _rows_cols(M, N, M, 1024, k)
        cc = torch.as_tensor(cols, device=DEV)
        check_product(C[:, cc], f64(X), f64(W[:, cc]), idx.cpu().numpy(), 1e-2)
    del X, W, ws
    torch.cuda.empty_cache()


def test_w8_decode_mlp_up_full_size():
    """The INT8-weight decode workload at full size, x[1×8192] · (Wq · diag(scale))
    with Wq int8 [8192×28672] and W's norms cached: scores against the
    dequantized weight in fp64, the selection bit-exact on the library's
    scores, the product on 1024 sampled columns."""
    X, _ = inputs.mlp_up(seed=0, device=DEV)
    X = X[:1].contiguous()
    Wq, sc = inputs.int8_weight(8192, 28672, std=0.01, seed=1, device=DEV)
    K, N = Wq.shape
    sc64 = sc.double().cpu().numpy()
    bn = rmm.b_norms_w8(Wq, sc)
    s = rmm.score_b_norms(X, bn)
    s_ref = _block_scores(X, lambda r0, r1: O.dequantize_w8(Wq[r0:r1].cpu().numpy(), sc64), K)
    check_scores(s.cpu().numpy(), s_ref)
    k = rmm.keep_count(0.5, K)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced_w8(X, Wq, sc, 0.5, b_norm=bn, idx_out=idx)
    rmm.check(ws)
    _check_selection_exact(s, idx, k)
    check_selection(idx.cpu().numpy(), s_ref, k)
    _, cols = _rows_cols(1, N, 1, 1024, 7)
    cc = torch.as_tensor(cols, device=DEV)
    W_sub = O.dequantize_w8(Wq[:, cc].cpu().numpy(), sc64[cols])
    check_product(C[:, cc], f64(X), W_sub, idx.cpu().numpy(), 1e-2)
    del X, Wq, sc, ws
    torch.cuda.empty_cache()


def test_decode_4096_full_size():
    """x[1×4096] · W[4096×4096] (1 % outlier channels, W's norms cached) through
    the fused call: all scores, the selection bit-exact on the library's
    scores, the whole product."""
    X, W = inputs.linear_projection(M=16, seed=0, device=DEV)
    X = X[:1].contiguous()
    K, N = W.shape
    bn = rmm.b_norms(W)
    s = rmm.score_b_norms(X, bn)
    s_ref = O.slice_scores(f64(X), f64(W))
    check_scores(s.cpu().numpy(), s_ref)
    k = rmm.keep_count(0.5, K)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced_b_norms(X, W, bn, 0.5, idx_out=idx)
    rmm.check(ws)
    _check_selection_exact(s, idx, k)
    check_selection(idx.cpu().numpy(), s_ref, k)
    check_product(C, f64(X), f64(W), idx.cpu().numpy(), 1e-2)


def test_w8_linear_4096_full_size():
    """X[4096×4096] · (Wq · diag(scale)), Wq int8 [4096×4096], W's norms cached:
    the pack + tensor-core GEMM route at full size — all scores against the
    dequantized weight, the selection bit-exact on the library's scores, the
    product on 128 sampled rows × 512 sampled columns."""
    X, _ = inputs.linear_projection(seed=0, device=DEV)
    Wq, sc = inputs.int8_weight(4096, 4096, std=0.02, seed=1, device=DEV)
    M, K = X.shape
    N = Wq.shape[1]
    sc64 = sc.double().cpu().numpy()
    bn = rmm.b_norms_w8(Wq, sc)
    s = rmm.score_b_norms(X, bn)
    W64 = O.dequantize_w8(Wq.cpu().numpy(), sc64)
    s_ref = O.slice_scores(f64(X), W64)
    check_scores(s.cpu().numpy(), s_ref)
    k = rmm.keep_count(0.5, K)
    idx = torch.empty(k, dtype=torch.int32, device=DEV)
    C, ws = rmm.matmul_reduced_w8(X, Wq, sc, 0.5, b_norm=bn, idx_out=idx)
    rmm.check(ws)
    _check_selection_exact(s, idx, k)
    check_selection(idx.cpu().numpy(), s_ref, k)
    rows, cols = _rows_cols(M, N, 128, 512, 11)
    rr, cc = torch.as_tensor(rows, device=DEV), torch.as_tensor(cols, device=DEV)
    # the pack route multiplies the weight rounded to bf16
    check_product(C[rr][:, cc], f64(X[rr]), W64[:, cols], idx.cpu().numpy(), 1e-2, w_rel=U_BF16)
    del X, Wq, sc, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("S", [8192, 32768])
def test_pv_softmax_long_context(S):
    """P·V with its softmax producer at full size (32 heads, d 128, logits
    3·N(0,1) stored bf16, causal): the stored P on sampled rows against the
    fp64 causal softmax, the producer's scores on sampled keys against the
    oracle's scores of that P, every head's selection bit-exact on the
    producer's scores, and 256 whole output rows of two heads against the
    oracle's product over the kept keys."""
    L, V = inputs.attention_logits(bh=32, S=S, d=128, seed=0, device=DEV)
    k = rmm.keep_count(0.5, S)
    idx = torch.empty(32, k, dtype=torch.int32, device=DEV)
    Oo, P, ws = rmm.pv_softmax_reduced(L, V, 0.5, idx_out=idx)
    rmm.check(ws)
    # the producer's own scores (its stage call rewrites the same P, bit for bit)
    P_before = P[5, S - 3].clone()
    stats = rmm.softmax_row_stats(L)
    _, s = rmm.softmax_score(L, stats, V, score=True, P=P)
    assert torch.equal(P[5, S - 3], P_before)
    for h in range(32):
        _check_selection_exact(s[h], idx[h], k)
    p_rel = 2.0 ** -8 + 2e-4 + 2.0 ** -8 * 2e-4
    for h in (0, 21):
        rows, cols = _rows_cols(S, S, 256, 1024, h + S)
        rr, cc = torch.as_tensor(rows, device=DEV), torch.as_tensor(cols, device=DEV)
        # P on sampled rows: softmax of the whole row (its visible part), masked entries zero
        L_rows = f64(L[h][rr])
        visible = np.arange(S)[None, :] <= rows[:, None]
        Lm = np.where(visible, L_rows, -np.inf)
        P_ref = np.exp(Lm - Lm.max(axis=1, keepdims=True))
        P_ref /= P_ref.sum(axis=1, keepdims=True)
        got = f64(P[h][rr])
        assert np.all(got[~visible] == 0)
        assert np.all(np.abs(got - P_ref) <= p_rel * P_ref + 1e-38)
        # scores of sampled keys from the whole stored columns of P
        s_ref = O.slice_scores(f64(P[h][:, cc]), f64(V[h][cc]))
        check_scores(s[h][cc].cpu().numpy(), s_ref)
        # whole output rows: O[r, :] = P[r, I] · V[I, :]
        check_product(Oo[h][rr], f64(P[h][rr]), f64(V[h]), idx[h].cpu().numpy(), 1e-2)
    del L, V, P, Oo, ws
    torch.cuda.empty_cache()
