"""Decode shapes whose score needs only A — B's row norms cached, or the
A-only score: with M <= 4 rows and K <= 8192 the fused call computes the
scores inside the selection kernel (2 launches), otherwise it runs the score
kernel first (3 launches). Either way the scores must be the bits the score
kernel writes (rmm_score_b_norms / rmm_score), the kept set the one
rmm_select picks from those scores, and the product must pass the oracle
check."""
import pytest
import torch

from input_adaptive_reduced_02_b200 import rmm
from tests._parity import check_single

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _scores_in_workspace(ws: rmm.Workspace, batch: int, K: int) -> torch.Tensor:
    """The fused call's scores: its workspace holds the status word in its
    first KiB and the [batch][K] f32 scores right after (the library's
    workspace layout, read here white-box)."""
    raw = ws._buf[ws.offset + 1024: ws.offset + 1024 + batch * K * 4]
    return raw.view(torch.float32).view(batch, K).clone()


def _x(batch, M, K, dtype, aligned, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    X = torch.randn(batch, M, K + 1, generator=g, device=DEV)
    X[:, :, ::97] *= 20.0  # a few outlier channels
    X = X.to(dtype)
    return X[:, :, :K].contiguous() if aligned else X[:, :, 1:]  # row pitch K + 1: no 16-byte loads


def _folded(M, K):
    return M <= 4 and K <= 8192


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("M,K,batch,aligned", [(1, 4100, 1, True), (3, 4100, 1, False), (4, 8192, 2, True),
                                               (2, 1000, 3, False), (1, 9000, 1, True), (16, 4100, 1, True)])
def test_decode_scores_inside_the_selection(dtype, M, K, batch, aligned):
    N = 1000  # K = 4100: the last thread's run of keys is partial
    X = _x(batch, M, K, dtype, aligned, seed=M * 10 + batch)
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    W = torch.randn(K, N, generator=g, device=DEV).to(dtype)
    Wb = W.unsqueeze(0).expand(batch, K, N)
    bn = rmm.b_norms(W)
    k = rmm.keep_count(0.5, K)
    idx = torch.empty(batch, k, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = rmm.launch_count()
    C, ws = rmm.matmul_reduced_b_norms(X, Wb, bn, 0.5, idx_out=idx)
    torch.cuda.synchronize()
    # select (with the scores) and gather-GEMV, or score, select, gather-GEMV
    assert rmm.launch_count() - n0 == (2 if _folded(M, K) else 3)
    rmm.check(ws)
    s_ref = rmm.score_b_norms(X, bn)
    assert torch.equal(_scores_in_workspace(ws, batch, K), s_ref.view(batch, K))
    assert torch.equal(idx, rmm.select(s_ref, k).view(batch, k))
    for b in range(batch):
        check_single(X[b], W, 0.5, "product", C[b], idx[b])


@pytest.mark.parametrize("M,batch", [(1, 1), (4, 2), (7, 2)])
def test_decode_a_only_scores_inside_the_selection(M, batch):
    K, N = 3000, 700
    X = _x(batch, M, K, torch.bfloat16, True, seed=41 + M)
    g = torch.Generator(device=DEV)
    g.manual_seed(6)
    W = torch.randn(K, N, generator=g, device=DEV).to(torch.bfloat16)
    Wb = W.unsqueeze(0).expand(batch, K, N)
    k = rmm.keep_count(0.3, K)
    idx = torch.empty(batch, k, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = rmm.launch_count()
    C, ws = rmm.matmul_reduced(X, Wb, 0.3, mode="a_only", idx_out=idx)
    torch.cuda.synchronize()
    assert rmm.launch_count() - n0 == (2 if _folded(M, K) else 3)
    rmm.check(ws)
    s_ref = rmm.score(X, Wb, mode="a_only")
    assert torch.equal(_scores_in_workspace(ws, batch, K), s_ref.view(batch, K))
    assert torch.equal(idx, rmm.select(s_ref, k).view(batch, k))
    for b in range(batch):
        check_single(X[b], W, 0.3, "a_only", C[b], idx[b])


def test_decode_scores_flag_non_finite_and_clear_the_status():
    """A NaN in x sets the non-finite bit through the folded selection, and a
    later call on the same workspace starts from a cleared status word (with
    one batch item the selection's only block clears it; with two, a memset)."""
    K, N = 2048, 512
    W = torch.randn(K, N, device=DEV).to(torch.bfloat16)
    bn = rmm.b_norms(W)
    for batch in (1, 2):
        X = _x(batch, 1, K, torch.bfloat16, True, seed=3)
        Wb = W.unsqueeze(0).expand(batch, K, N)
        Xbad = X.clone()
        Xbad[-1, 0, 17] = float("nan")
        _, ws = rmm.matmul_reduced_b_norms(Xbad, Wb, bn, 0.5)
        _, ws = rmm.matmul_reduced_b_norms(X, Wb, bn, 0.5, workspace=ws)
        rmm.check(ws)  # the clean call cleared the bit the previous call left
        _, ws = rmm.matmul_reduced_b_norms(Xbad, Wb, bn, 0.5, workspace=ws)
        with pytest.raises(rmm.RMMError):
            rmm.check(ws)
