"""Debug checks (rmm_set_debug): a stage call handed a kept-index list with an
entry outside [0, K) validates the list on the device and returns
RMM_ERR_INVALID before any kernel reads through it; valid lists give the
same bits as without the checks; the fused call reports a non-finite score
from the call itself. No out-of-range index ever reaches a kernel that reads
through it: the check runs first and the stage call stops on its result."""
from __future__ import annotations

import pytest
import torch

from input_adaptive_reduced_02_b200 import inputs, rmm

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture
def debug():
    prev = rmm.set_debug(True)
    yield
    rmm.set_debug(prev)


def _ab(M, K, N, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    A = torch.randn(M, K, generator=g, device=DEV).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g, device=DEV).to(torch.bfloat16)
    return A, B


def test_valid_indices_pass_and_match_the_unchecked_calls(debug):
    A, B = _ab(200, 600, 300, 1)
    idx = rmm.select(rmm.score(A, B), 300)
    A_S, B_S = rmm.pack(A, B, idx)
    C = rmm.gemv_gather(A[:4].contiguous(), B, idx)
    rmm.set_debug(False)
    A_S2, B_S2 = rmm.pack(A, B, idx)
    assert torch.equal(A_S, A_S2) and torch.equal(B_S, B_S2)
    assert torch.equal(C, rmm.gemv_gather(A[:4].contiguous(), B, idx))


@pytest.mark.parametrize("bad", [-1, 600, 2 ** 31 - 1])
def test_out_of_range_index_is_refused_before_any_read(debug, bad):
    A, B = _ab(64, 600, 96, 2)
    idx = rmm.select(rmm.score(A, B), 300)
    idx[137] = bad
    n0 = rmm.launch_count()
    with pytest.raises(rmm.RMMError) as e:
        rmm.pack(A, B, idx)
    assert e.value.status == rmm.RMM_ERR_INVALID
    assert "idx[0][137]" in str(e.value) and str(bad) in str(e.value)
    assert rmm.launch_count() - n0 == 1  # the check kernel only
    with pytest.raises(rmm.RMMError) as e:
        rmm.gemv_gather(A[:2].contiguous(), B, idx)
    assert e.value.status == rmm.RMM_ERR_INVALID
    Wq, scale = inputs.int8_weight(600, 96, seed=3, device=DEV)
    with pytest.raises(rmm.RMMError):
        rmm.pack_w8(A, Wq, scale, idx)
    with pytest.raises(rmm.RMMError):
        rmm.gemv_gather_w8(A[:2].contiguous(), Wq, scale, idx)
    # the context is intact: a valid call still works
    idx[137] = 0 if bad != 0 else 1
    rmm.pack(A, B, rmm.select(rmm.score(A, B), 300))
    torch.cuda.synchronize()


def test_batched_index_position_is_reported(debug):
    g = torch.Generator(device=DEV)
    g.manual_seed(4)
    A = torch.randn(3, 32, 200, generator=g, device=DEV).to(torch.bfloat16)
    B = torch.randn(3, 200, 40, generator=g, device=DEV).to(torch.bfloat16)
    idx = rmm.select(rmm.score(A, B), 50)
    idx[2, 7] = -5
    with pytest.raises(rmm.RMMError) as e:
        rmm.pack(A, B, idx)
    assert "idx[2][7] = -5" in str(e.value)


def test_fused_call_reports_nonfinite_directly(debug):
    A, B = _ab(64, 128, 64, 5)
    A[3, 17] = float("nan")
    with pytest.raises(rmm.RMMError) as e:
        rmm.matmul_reduced(A, B, 0.5)
    assert e.value.status == rmm.RMM_ERR_NONFINITE
