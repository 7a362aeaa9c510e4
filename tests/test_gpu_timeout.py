"""The tensor-core GEMM's bounded waits: with the TMA producer idled by the test
hook, the MMA and epilogue waits run out after the configured limit, the kernel
records RMM_STATUS_BIT_TIMEOUT, drains, frees tensor memory and returns. No
fault and no trap: the context stays usable and the next call is correct."""
from __future__ import annotations

import pytest
import torch

from input_adaptive_reduced_02_b200 import rmm

from _parity import check_product, f64

pytestmark = pytest.mark.gpu


def test_stalled_producer_times_out_and_context_survives():
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    A = torch.randn(512, 256, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(256, 640, generator=g, device="cuda").to(torch.bfloat16)
    s = rmm.score(A, B)
    k = rmm.keep_count(0.5, 256)
    idx = rmm.select(s, k)
    A_S, B_S = rmm.pack(A, B, idx)
    torch.cuda.synchronize()

    status = rmm.status_word()
    rmm.set_wait_limit_ns(20_000_000)  # 20 ms per wait
    rmm.set_stall_producer_for_test(True)
    try:
        rmm.gemm(A_S, B_S, k, status=status)
        torch.cuda.synchronize()
    finally:
        rmm.set_stall_producer_for_test(False)
        rmm.set_wait_limit_ns(0)
    with pytest.raises(rmm.RMMError) as e:
        rmm.check(status)
    assert e.value.status == rmm.RMM_ERR_TIMEOUT

    C = rmm.gemm(A_S, B_S, k, status=status)
    rmm.check(status)
    check_product(C, f64(A), f64(B), idx.cpu().numpy(), 1e-2)
