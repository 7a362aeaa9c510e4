"""P·V with its softmax producer ("Escopo de Aplicação": P·V reduced over the
keys; P = softmax of the scaled logits): the row statistics and the stored P
against the fp64 oracle's causal softmax, the key scores the producer
accumulates against the oracle's scores of that P, and the fused call's
selection and product against the oracle, on ragged and aligned sizes, with
and without the causal mask, bf16 and f32 logits.

Tolerance on P: the library forms p = exp2(x - max)·(1/sum) in f32 (x the
scaled logit; the sum over at most 32768 terms errs by well under 2e-4
relative) and rounds to bf16 (2^-8 relative), so |P - P_exact| <=
(2^-8 + 2e-4 + 2^-8·2e-4)·P_exact; masked entries are exactly 0."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O
from input_adaptive_reduced_02_b200 import inputs, rmm

from _parity import check_product, check_scores, check_selection, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"
P_REL = 2.0 ** -8 + 2e-4 + 2.0 ** -8 * 2e-4


def _check_P(P_gpu: torch.Tensor, L: torch.Tensor, scale: float, causal: bool):
    P64 = O.causal_softmax(f64(L), scale, causal)
    got = f64(P_gpu)
    assert np.all(got[P64 == 0] == 0), "masked entries must be exactly zero"
    assert np.all(np.abs(got - P64) <= P_REL * P64 + 1e-38), \
        f"P off the softmax by {np.max(np.abs(got - P64) / np.maximum(P64, 1e-38)):.3e} relative"


CASES = [  # bh, S_q, S_k, d, logits dtype, scale, causal
    (2, 300, 300, 64, torch.bfloat16, 1.0, True),     # ragged: scalar paths, a partial last strip
    (3, 1024, 1024, 128, torch.bfloat16, 1.0, True),  # 16-byte paths
    (2, 200, 512, 128, torch.bfloat16, 0.125, True),  # fewer queries than keys, a scale
    (2, 256, 384, 72, torch.bfloat16, 1.0, False),    # no mask; d not a multiple of 8 for V
    (2, 512, 512, 128, torch.float32, 1.0, True),     # f32 logits
    (2, 200, 200, 64, torch.bfloat16, 1.0, True),     # 16-byte rows, a partial last strip (200 % 128)
    (1, 136, 392, 128, torch.bfloat16, 1.0, True),    # the same with fewer queries than keys
    (2, 96, 200, 64, torch.float32, 1.0, False),      # f32 logits, a partial last strip, no mask
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}x{c[3]}-{str(c[4])[6:]}-s{c[5]}-c{int(c[6])}")
def test_softmax_producer_and_scores(case):
    bh, S_q, S_k, d, ldt, scale, causal = case
    L, V = inputs.attention_logits(bh, S_k, d, seed=bh + S_k, device=DEV, dtype=ldt, S_q=S_q)
    stats = rmm.softmax_row_stats(L, scale, causal)
    P, s = rmm.softmax_score(L, stats, V, scale, causal)
    _check_P(P, L, scale, causal)
    P_only, none = rmm.softmax_score(L, stats, V, scale, causal, score=False)
    assert none is None and torch.equal(P_only, P)
    _, s_a = rmm.softmax_score(L, stats, None, scale, causal)
    for h in range(bh):
        P64 = f64(P[h])
        check_scores(s[h].cpu().numpy(), O.slice_scores(P64, f64(V[h])))
        check_scores(s_a[h].cpu().numpy(), O.slice_scores(P64, None, "a_only"))


@pytest.mark.parametrize("case", [c for c in CASES if c[2] % 8 == 0],
                         ids=lambda c: f"{c[0]}x{c[1]}x{c[2]}x{c[3]}-c{int(c[6])}")
@pytest.mark.parametrize("rho", [0.3, 0.5, 1.0])
def test_fused_softmax_pv_matches_the_oracle(case, rho):
    bh, S_q, S_k, d, ldt, scale, causal = case
    L, V = inputs.attention_logits(bh, S_k, d, seed=7 + S_q, device=DEV, dtype=ldt, S_q=S_q)
    k = rmm.keep_count(rho, S_k)
    idx = torch.empty(bh, k, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    n0 = rmm.launch_count()
    Oo, P, ws = rmm.pv_softmax_reduced(L, V, rho, scale, causal, idx_out=idx)
    torch.cuda.synchronize()
    assert rmm.launch_count() - n0 == 5  # row stats, softmax + score, select, mask, gemm
    rmm.check(ws)
    _check_P(P, L, scale, causal)
    for h in range(bh):
        P64, V64 = f64(P[h]), f64(V[h])
        check_selection(idx[h].cpu().numpy(), O.slice_scores(P64, V64), k)
        check_product(Oo[h], P64, V64, idx[h].cpu().numpy(), 1e-2)
    # the stage calls give the same bits
    stats = rmm.softmax_row_stats(L, scale, causal)
    P2, s2 = rmm.softmax_score(L, stats, V, scale, causal)
    idx2 = rmm.select(s2, k)
    O2 = rmm.gemm_full(P2, rmm.mask_rows(V, idx2), d, causal_off=(S_k - S_q) if causal else -1)
    assert torch.equal(P2, P) and torch.equal(idx2, idx) and torch.equal(O2, Oo)
    if causal:  # the dense GEMM over the same P (zeros above the mask included) gives the same product
        O3 = rmm.gemm_full(P2, rmm.mask_rows(V, idx2), d)
        for h in range(bh):
            check_product(O3[h], f64(P[h]), f64(V[h]), idx[h].cpu().numpy(), 1e-2)


def test_oracle_pipeline_end_to_end_small():
    """The whole fused call against the oracle's pipeline in the pages' order on
    the same logits; the selections agree up to near-ties of the scores."""
    L, V = inputs.attention_logits(2, 256, 64, seed=3, device=DEV)
    Oo, P, ws = rmm.pv_softmax_reduced(L, V, 0.5, idx_out=(idx := torch.empty(2, 128, dtype=torch.int32, device=DEV)))
    rmm.check(ws)
    O_ref, idx_ref, s_ref, P_ref = O.pv_softmax_reduced(f64(L), f64(V), 0.5)
    # P agrees with the oracle's stored P except where f32 rounding moved a value across a bf16 halfway point
    diff = f64(P) != P_ref
    assert diff.mean() < 0.01
    for h in range(2):
        check_selection(idx[h].cpu().numpy(), O.slice_scores(f64(P[h]), f64(V[h])), 128)
        check_product(Oo[h], f64(P[h]), f64(V[h]), idx[h].cpu().numpy(), 1e-2)


def test_nonfinite_logits_are_reported():
    L, V = inputs.attention_logits(1, 128, 64, seed=4, device=DEV)
    L[0, 77, 3] = float("nan")
    Oo, P, ws = rmm.pv_softmax_reduced(L, V, 0.5)
    with pytest.raises(rmm.RMMError) as e:
        rmm.check(ws)
    assert e.value.status == rmm.RMM_ERR_NONFINITE


def test_fused_softmax_pv_argument_checks():
    L, V = inputs.attention_logits(1, 100, 64, seed=5, device=DEV)  # S_k = 100: not a multiple of 8
    with pytest.raises(rmm.RMMError) as e:
        rmm.pv_softmax_reduced(L, V, 0.5)
    assert e.value.status == rmm.RMM_ERR_UNSUPPORTED
    L2, V2 = inputs.attention_logits(1, 64, 64, seed=6, device=DEV, S_q=128)  # more queries than keys
    with pytest.raises(rmm.RMMError) as e:
        rmm.softmax_row_stats(L2, causal=True)
    assert e.value.status == rmm.RMM_ERR_INVALID
