"""The parity harness itself, on the CPU: a product computed correctly in f32
(the library's accumulation precision) passes the element-wise bound, and
plausible localised faults of a GPU kernel fail it even where the whole-matrix
Frobenius tolerance would let them through: one wrong 32 x 32 tile, a tile
whose split-K partial sum went missing, one column of C holding its
neighbour's values, one kept slice left out, a single NaN. A kept-index list
with an index outside [0, K) (which NumPy would wrap around) or a repeated
index is rejected too."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import rmm_oracle as O

from _parity import check_index_list, check_product, check_selection, f64

M, K, N = 512, 1024, 512


@pytest.fixture(scope="module")
def case():
    g = torch.Generator().manual_seed(7)
    A = (torch.randn(M, K, generator=g) * torch.exp(torch.randn(K, generator=g))).to(torch.bfloat16)
    B = torch.randn(K, N, generator=g).to(torch.bfloat16)
    A64, B64 = f64(A), f64(B)
    s = O.slice_scores(A64, B64)
    k = O.keep_count(0.5, K)
    idx = O.select_top(s, k)
    ii = torch.as_tensor(idx)
    # the product over the kept slices accumulated in f32, as the library does
    C32 = A[:, ii].float() @ B[ii, :].float()
    return A64, B64, s, k, idx, C32


def test_f32_product_passes(case):
    A64, B64, s, k, idx, C32 = case
    err = check_product(C32, A64, B64, idx, 1e-2)
    assert err < 1e-5


def test_bf16_output_passes_only_with_its_rounding_term(case):
    A64, B64, s, k, idx, C32 = case
    C16 = C32.to(torch.bfloat16)
    check_product(C16, A64, B64, idx, 1e-2)
    # the same values declared as f32 output exceed the f32 bound
    with pytest.raises(AssertionError, match="forward-error bound"):
        check_product(f64(C16), A64, B64, idx, 1e-2, out_dtype=torch.float32)


def _corrupt(C32, how):
    C = C32.clone()
    if how == "zero_tile":
        C[64:96, 32:64] = 0.0
    elif how == "half_tile":  # one split-K half missing from its reduce-add
        C[128:160, 96:128] *= 0.5
    elif how == "neighbour_column":
        C[:, 17] = C[:, 18]
    elif how == "nan":
        C[3, 5] = float("nan")
    elif how == "transposed_tile":
        C[0:32, 0:32] = C[0:32, 0:32].t().clone()
    return C


@pytest.mark.parametrize("how", ["zero_tile", "half_tile", "neighbour_column", "nan", "transposed_tile"])
def test_localised_faults_fail(case, how):
    A64, B64, s, k, idx, C32 = case
    C = _corrupt(C32, how)
    if how != "nan":
        # small enough for the whole-matrix norm alone to let it through
        assert O.frobenius_rel_error(f64(C), O.reduced_product(A64, B64, idx)) < 1e-1
    with pytest.raises(AssertionError):
        check_product(C, A64, B64, idx, 1e-1)


def test_one_missing_kept_slice_fails(case):
    A64, B64, s, k, idx, C32 = case
    t = int(idx[k // 2])
    C = C32 - torch.outer(torch.as_tensor(A64[:, t], dtype=torch.float32),
                          torch.as_tensor(B64[t, :], dtype=torch.float32))
    assert O.frobenius_rel_error(f64(C), O.reduced_product(A64, B64, idx)) < 1e-1
    with pytest.raises(AssertionError, match="forward-error bound"):
        check_product(C, A64, B64, idx, 1e-1)


@pytest.mark.parametrize("bad", ["negative", "past_end", "repeated"])
def test_index_lists_out_of_range_or_repeated_fail(case, bad):
    A64, B64, s, k, idx, C32 = case
    wrong = idx.copy()
    if bad == "negative":
        wrong[0] = -1
    elif bad == "past_end":
        wrong[-1] = K
    else:
        wrong[1] = wrong[0]
    with pytest.raises(AssertionError):
        check_index_list(wrong, K, k)
    with pytest.raises(AssertionError):
        check_selection(wrong, s, k)
    with pytest.raises((AssertionError, IndexError)):
        check_product(C32, A64, B64, wrong, 1e-2)
    ok, _ = O.selection_matches(wrong, idx, s)
    assert not ok
