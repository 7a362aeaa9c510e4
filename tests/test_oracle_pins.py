"""Pins for the fp64 oracle: each test checks the oracle against something other
than itself — hand-worked closed forms, exact integer arithmetic, brute force
over every subset, or an inequality the mathematics fixes.

The method is the one on the summary pages of "Reduced Matrix Multiplication:
Input-Adaptive Matrix-Product Reduction for LLM Inference" (gist.science,
Resumo Técnico › Metodologia: "Mecanismo Central", "Estratégia de Seleção",
"Base Teórica").
"""
from __future__ import annotations

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import rmm_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rmm_hand_examples.json")


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


# ---------------------------------------------------------------- golden cases
@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    A = np.array(case["A"], dtype=np.float64)
    if case["kind"] == "qk":
        B = np.array(case["Kmat"], dtype=np.float64).T
    else:
        B = np.array(case["B"], dtype=np.float64)
    for mode, want in case["scores"].items():
        got = O.slice_scores(A, B, mode)
        np.testing.assert_allclose(got, np.array(want, dtype=np.float64), rtol=1e-15, atol=0)
    for r in case["results"]:
        assert O.keep_count(r["rho"], A.shape[1]) == r["k_keep"]
        C, idx, _ = O.matmul_reduced(A, B, r["rho"], r["mode"])
        assert idx.tolist() == r["idx"], (r, idx)
        np.testing.assert_array_equal(C, np.array(r["C"], dtype=np.float64))
        if case["kind"] == "qk":
            Cq, idxq, _ = O.qk_reduced(A[None], np.array(case["Kmat"], dtype=np.float64)[None],
                                       r["rho"], r["mode"])
            assert idxq[0].tolist() == r["idx"]
            np.testing.assert_array_equal(Cq[0], np.array(r["C"], dtype=np.float64))


# ---------------------------------------------------------------- keep count
CONFIG_K = [256, 4096, 128, 8192, 16384, 32768, 28672]
RHOS = [0.1, 0.2, 0.25, 0.3, 0.4, 0.5, 0.6, 0.7, 0.75, 0.8, 0.9, 1.0]


def test_keep_count_equals_exact_decimal_ceiling():
    """k = ceil(rho*d) with rho read as the decimal the user wrote: the double
    product agrees with exact rational arithmetic on every workload K and on
    all K < 2048."""
    for K in CONFIG_K + list(range(1, 2048)):
        for rho in RHOS:
            exact = math.ceil(Fraction(str(rho)) * K)
            assert O.keep_count(rho, K) == exact, (rho, K)


def test_keep_count_domain():
    assert O.keep_count(1e-9, 10) == 1
    assert O.keep_count(1.0, 7) == 7
    for bad in (0.0, -0.5, 1.0000001, float("nan")):
        with pytest.raises(ValueError):
            O.keep_count(bad, 10)
    with pytest.raises(ValueError):
        O.keep_count(0.5, 0)


# ---------------------------------------------------------------- scores
def test_score_closed_forms():
    # column (3,4) has norm 5; a one-hot row of B has the norm of its entry.
    A = np.zeros((5, 3))
    A[1, 0], A[4, 0] = 3.0, 4.0
    A[2, 1] = -7.0
    B = np.zeros((3, 4))
    B[0, 3] = -2.0
    B[1, 0], B[1, 1] = 1.0, 1.0
    B[2, 2] = 9.0
    np.testing.assert_allclose(O.column_norms(A), [5.0, 7.0, 0.0], rtol=1e-15)
    np.testing.assert_allclose(O.row_norms(B), [2.0, math.sqrt(2.0), 9.0], rtol=1e-15)
    np.testing.assert_allclose(O.slice_scores(A, B, O.SCORE_PRODUCT),
                               [10.0, 7.0 * math.sqrt(2.0), 0.0], rtol=1e-15)
    np.testing.assert_allclose(O.slice_scores(A, B, O.SCORE_A_ONLY), [5.0, 7.0, 0.0], rtol=1e-15)


def test_score_uses_columns_of_A_and_rows_of_B_nonsquare():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((3, 7))
    B = rng.standard_normal((7, 5))
    s = O.slice_scores(A, B)
    for k in range(7):
        a = math.sqrt(sum(A[i, k] ** 2 for i in range(3)))
        b = math.sqrt(sum(B[k, j] ** 2 for j in range(5)))
        assert abs(s[k] - a * b) <= 1e-14 * a * b


# ---------------------------------------------------------------- exact identities
def _int_matrix(rng, shape, lo=-9, hi=10):
    return rng.integers(lo, hi, size=shape).astype(np.int64)


def _exact_product(A, B, ks):
    """Σ_{k in ks} A[:, k] ⊗ B[k, :] with Python integers (exact)."""
    M, N = A.shape[0], B.shape[1]
    out = [[0] * N for _ in range(M)]
    for k in ks:
        for i in range(M):
            a = int(A[i, k])
            if a:
                for j in range(N):
                    out[i][j] += a * int(B[k, j])
    return np.array(out, dtype=np.int64)


def test_rho_one_is_the_full_product_exactly():
    rng = np.random.default_rng(2)
    for M, K, N in [(3, 5, 4), (7, 13, 2), (1, 9, 6), (6, 1, 3)]:
        A, B = _int_matrix(rng, (M, K)), _int_matrix(rng, (K, N))
        C, idx, _ = O.matmul_reduced(A, B, 1.0)
        assert idx.tolist() == list(range(K))
        np.testing.assert_array_equal(C, _exact_product(A, B, range(K)).astype(np.float64))


@pytest.mark.parametrize("rho", [0.2, 0.5, 0.7, 0.9])
def test_kept_plus_dropped_is_the_full_product(rho):
    rng = np.random.default_rng(3)
    for M, K, N in [(4, 11, 5), (9, 16, 3), (2, 7, 8)]:
        A, B = _int_matrix(rng, (M, K)), _int_matrix(rng, (K, N))
        C, idx, _ = O.matmul_reduced(A, B, rho)
        dropped = sorted(set(range(K)) - set(idx.tolist()))
        full = _exact_product(A, B, range(K))
        rest = _exact_product(A, B, dropped)
        np.testing.assert_array_equal(C, (full - rest).astype(np.float64))


@pytest.mark.parametrize("mode", [O.SCORE_PRODUCT, O.SCORE_A_ONLY])
def test_error_bound_triangle_inequality(mode):
    rng = np.random.default_rng(4)
    for trial in range(20):
        M, K, N = rng.integers(1, 30, size=3)
        A = rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))[None, :]
        B = rng.standard_normal((K, N)) * np.exp(rng.standard_normal(K))[:, None]
        rho = float(rng.choice([0.1, 0.3, 0.5, 0.8]))
        C, idx, _ = O.matmul_reduced(A, B, rho, mode)
        dropped = np.setdiff1d(np.arange(K), idx)
        bound = sum(np.linalg.norm(A[:, k]) * np.linalg.norm(B[k, :]) for k in dropped)
        err = np.linalg.norm(A @ B - C)
        assert err <= bound * (1 + 1e-12) + 1e-12


def test_identity_weight_zeroes_dropped_columns():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((6, 10))
    B = np.eye(10)
    for rho in (0.3, 0.5, 1.0):
        C, idx, s = O.matmul_reduced(A, B, rho)
        expect = A.copy()
        expect[:, np.setdiff1d(np.arange(10), idx)] = 0.0
        np.testing.assert_array_equal(C, expect)
        # with B = I every row norm is 1, so the product score is the column norm
        np.testing.assert_array_equal(s, O.column_norms(A))


# ---------------------------------------------------------------- selection
def _lex_best_subset(s, k_keep):
    """Brute force: among all kept sets of size k_keep minimising the error bound
    Σ_{dropped} s_k, the one whose sorted index list is lexicographically lowest."""
    K = len(s)
    best = None
    for kept in itertools.combinations(range(K), k_keep):
        dropped_sum = sum(Fraction(s[k]) for k in range(K) if k not in kept)
        key = (dropped_sum, kept)
        if best is None or key < best:
            best = key
    return list(best[1]), best[0]


def test_bruteforce_topk_minimises_bound_and_breaks_ties_low():
    rng = np.random.default_rng(6)
    for trial in range(60):
        K = int(rng.integers(1, 11))
        # small integer scores produce many ties, including zeros
        s = rng.integers(0, 4, size=K).astype(np.float64)
        k_keep = int(rng.integers(1, K + 1))
        want, _ = _lex_best_subset(s, k_keep)
        assert O.select_top(s, k_keep).tolist() == want, (s, k_keep)


def test_bruteforce_topk_distinct_scores():
    rng = np.random.default_rng(7)
    for trial in range(40):
        K = int(rng.integers(1, 12))
        s = rng.random(K)
        k_keep = int(rng.integers(1, K + 1))
        want, _ = _lex_best_subset(s, k_keep)
        assert O.select_top(s, k_keep).tolist() == want


def test_zero_slices_are_dropped_first():
    rng = np.random.default_rng(8)
    A = rng.standard_normal((5, 12))
    B = rng.standard_normal((12, 4))
    A[:, [1, 6]] = 0.0   # zero activation columns
    B[[3, 9], :] = 0.0   # zero weight rows
    zero = {1, 3, 6, 9}
    for k_keep in range(1, 13):
        idx = O.select_top(O.slice_scores(A, B), k_keep).tolist()
        if k_keep <= 8:
            assert not (set(idx) & zero)
        else:
            # every nonzero slice is kept; zero slices fill in by ascending index
            assert set(range(12)) - zero <= set(idx)
            assert sorted(set(idx) & zero) == sorted(zero)[: k_keep - 8]


def test_equal_row_norms_give_the_same_selection_in_both_modes():
    rng = np.random.default_rng(9)
    A = rng.standard_normal((8, 20)) * np.exp(rng.standard_normal(20))[None, :]
    B = rng.standard_normal((20, 6))
    B /= np.linalg.norm(B, axis=1, keepdims=True)
    B *= 3.5
    for rho in (0.2, 0.5, 0.75):
        k = O.keep_count(rho, 20)
        a = O.select_top(O.slice_scores(A, B, O.SCORE_PRODUCT), k)
        b = O.select_top(O.slice_scores(A, B, O.SCORE_A_ONLY), k)
        assert a.tolist() == b.tolist()


def test_selection_rejects_nonfinite():
    with pytest.raises(FloatingPointError):
        O.select_top(np.array([1.0, np.nan, 2.0]), 1)
    with pytest.raises(FloatingPointError):
        O.select_top(np.array([1.0, np.inf, 2.0]), 1)


# ---------------------------------------------------------------- minimax reading
def test_minimax_statement_by_construction():
    """'Base Teórica': with only A known, top-k by column norm minimises the
    worst case over B (‖B‖₂ ≤ 1) of ‖A·B − A_S·B_S‖_F = ‖A_D·B_D‖_F, whose value
    is ‖A_D‖_F. Check the worst case is attained (orthonormal rows) and never
    exceeded (random contractions), then that the a_only top-k minimises it."""
    rng = np.random.default_rng(10)
    M, K, N = 4, 7, 9
    A = rng.standard_normal((M, K)) * np.exp(rng.standard_normal(K))[None, :]
    for k_keep in range(1, K):
        worst = {}
        for kept in itertools.combinations(range(K), k_keep):
            D = [k for k in range(K) if k not in kept]
            AD = A[:, D]
            wc = math.sqrt(sum(AD[i, j] ** 2 for i in range(M) for j in range(len(D))))
            # attained: B with orthonormal rows (‖B‖₂ = 1)
            Q, _ = np.linalg.qr(rng.standard_normal((N, K)))
            Bo = Q.T  # K×N, orthonormal rows
            err = np.linalg.norm(AD @ Bo[D, :])
            assert abs(err - wc) <= 1e-12 * max(1.0, wc)
            # never exceeded by a random B scaled to spectral norm 1
            for _ in range(3):
                Br = rng.standard_normal((K, N))
                Br /= np.linalg.norm(Br, 2)
                assert np.linalg.norm(AD @ Br[D, :]) <= wc * (1 + 1e-12)
            worst[kept] = wc
        best = min(worst.values())
        idx = O.select_top(O.slice_scores(A, np.ones((K, 1)), O.SCORE_A_ONLY), k_keep)
        assert worst[tuple(idx.tolist())] <= best * (1 + 1e-12)


# ---------------------------------------------------------------- batched sites
def test_batched_sites_select_per_item():
    rng = np.random.default_rng(11)
    Q = rng.standard_normal((3, 5, 8))
    Km = rng.standard_normal((3, 6, 8))
    C, idx, s = O.qk_reduced(Q, Km, 0.5)
    for b in range(3):
        C1, idx1, _ = O.matmul_reduced(Q[b], Km[b].T, 0.5)
        assert idx[b].tolist() == idx1.tolist()
        np.testing.assert_array_equal(C[b], C1)
        # column k of Km is row k of B = Kmᵀ
        for k in range(8):
            assert abs(s[b, k] - np.linalg.norm(Q[b][:, k]) * np.linalg.norm(Km[b][:, k])) < 1e-12
    P = rng.random((2, 6, 6))
    V = rng.standard_normal((2, 6, 4))
    C, idx, _ = O.pv_reduced(P, V, 0.5)
    assert C.shape == (2, 6, 4) and idx.shape == (2, 3)


def test_pv_site_closed_form_with_permutation_attention():
    """P·V reduces over keys: with each query q attending to key π(q) alone
    (a permutation that is not its own inverse, so P ≠ Pᵀ) every key column
    of P has norm 1, key k scores ‖V[k,:]‖, the kept keys are the rows of V
    with the largest norms, and row q of the output is V[π(q)] when key π(q)
    is kept and zero otherwise. Two heads with different V select
    differently."""
    S, d = 6, 3
    perm = (np.arange(S) + 2) % S
    P1 = np.zeros((S, S))
    P1[np.arange(S), perm] = 1.0
    P = np.stack([P1, P1])
    V = np.zeros((2, S, d))
    V[0, :, 0] = [1.0, 5.0, 2.0, 6.0, 3.0, 4.0]
    V[1, :, 0] = [6.0, 1.0, 5.0, 2.0, 4.0, 3.0]
    V[:, :, 2] = np.arange(S)
    # row norms: head 0: 1, √26, √8, √45, 5, √41 -> keys {1, 3, 5};
    #            head 1: 6, √2, √29, √13, √32, √34 -> keys {0, 4, 5}
    norms = [np.sqrt([1.0, 26.0, 8.0, 45.0, 25.0, 41.0]), np.sqrt([36.0, 2.0, 29.0, 13.0, 32.0, 34.0])]
    keep = [[1, 3, 5], [0, 4, 5]]
    C, idx, s = O.pv_reduced(P, V, 0.5)
    for h in range(2):
        np.testing.assert_allclose(s[h], norms[h], rtol=1e-15)
        assert idx[h].tolist() == keep[h]
        expect = np.zeros((S, d))
        for q in range(S):
            if perm[q] in idx[h]:
                expect[q] = V[h][perm[q]]
        np.testing.assert_array_equal(C[h], expect)
    assert idx[0].tolist() != idx[1].tolist()


def test_selection_matches_window_rule():
    s = np.array([1.0, 2.0, 2.0 + 1e-7, 3.0])
    o = O.select_top(s, 2)  # {2, 3}
    ok, n = O.selection_matches(np.array([1, 3]), o, s)
    assert ok and n == 2
    ok, _ = O.selection_matches(np.array([0, 3]), o, s)
    assert not ok
    # the window is relative to the threshold score t: a gap of 1 at t = 1e6
    # (1e-6 relative) is a near-tie, a gap of 1e-6 at t = 1e-3 (1e-3 relative) is not
    big = np.array([5.0e5, 1.0e6, 1.0e6 + 1.0, 3.0e6])
    ok, n = O.selection_matches(np.array([1, 3]), O.select_top(big, 2), big)
    assert ok and n == 2
    small = np.array([5.0e-4, 1.0e-3, 1.0e-3 + 1.0e-6, 3.0e-3])
    ok, _ = O.selection_matches(np.array([1, 3]), O.select_top(small, 2), small)
    assert not ok


def test_kept_indices_must_lie_in_the_contraction_range():
    """I is a subset of {0, ..., K-1} ("Mecanismo Central"): an index of -1
    (which NumPy indexing would wrap to K-1), an index K or a repeated index
    is never a valid selection, even when the scores there are near-ties."""
    s = np.array([1.0, 1.0, 1.0, 1.0])  # every index a near-tie of every other
    o = O.select_top(s, 2)
    assert O.selection_matches(np.array([0, 1]), o, s) == (True, 0)
    for bad in ([-1, 0], [0, 4], [1, 1]):
        ok, _ = O.selection_matches(np.array(bad), o, s)
        assert not ok, bad
    A = np.arange(8.0).reshape(2, 4)
    B = np.ones((4, 3))
    with pytest.raises(IndexError):
        O.reduced_product(A, B, np.array([-1, 2]))
    with pytest.raises(IndexError):
        O.reduced_product(A, B, np.array([0, 4]))
    assert np.array_equal(O.reduced_product(A, B, np.array([1, 3])), np.array([[4.0] * 3, [12.0] * 3]))


def test_frobenius_rel_error():
    a = np.array([[3.0, 4.0]])
    assert O.frobenius_rel_error(a, a) == 0.0
    assert abs(O.frobenius_rel_error(np.zeros_like(a), a) - 1.0) < 1e-15


# ---------------------------------------------------------------- INT8 weights
def test_w8_hand_worked_example():
    """Per-output-channel INT8 weight, worked by hand: W = Wq · diag(scale) =
    [[1, 2], [1.5, -8], [-0.5, 0]]; column norms of A are (5, 0, 1), row norms
    of W (√5, √66.25, 0.5); product scores (5√5, 0, 0.5); ρ = 2/3 keeps {0, 2}
    and C = A[:, {0,2}]·W[{0,2}, :] = [[2.5, 6], [4, 8]]."""
    A = np.array([[3.0, 0.0, 1.0], [4.0, 0.0, 0.0]])
    Wq = np.array([[2, 1], [3, -4], [-1, 0]], dtype=np.int8)
    scale = np.array([0.5, 2.0])
    W = O.dequantize_w8(Wq, scale)
    assert np.array_equal(W, np.array([[1.0, 2.0], [1.5, -8.0], [-0.5, 0.0]]))
    s = O.slice_scores(A, W)
    assert np.allclose(s, [5.0 * math.sqrt(5.0), 0.0, 0.5], rtol=0, atol=1e-15)
    C, idx, _ = O.matmul_reduced_w8(A, Wq, scale, 2.0 / 3.0)
    assert idx.tolist() == [0, 2]
    assert np.array_equal(C, np.array([[2.5, 6.0], [4.0, 8.0]]))


def test_w8_unit_scales_reduce_to_the_integer_weight():
    rng = np.random.default_rng(7)
    A = rng.integers(-9, 10, size=(5, 12)).astype(np.float64)
    Wq = rng.integers(-127, 128, size=(12, 7)).astype(np.int8)
    C8, i8, _ = O.matmul_reduced_w8(A, Wq, np.ones(7), 0.5)
    C, i, _ = O.matmul_reduced(A, Wq.astype(np.float64), 0.5)
    assert np.array_equal(i8, i) and np.array_equal(C8, C)


def test_w8_uniform_scale_keeps_the_selection_and_scales_the_product():
    rng = np.random.default_rng(8)
    A = rng.standard_normal((6, 20))
    Wq = rng.integers(-127, 128, size=(20, 9)).astype(np.int8)
    C1, i1, _ = O.matmul_reduced_w8(A, Wq, np.full(9, 1.0), 0.4)
    C4, i4, _ = O.matmul_reduced_w8(A, Wq, np.full(9, 4.0), 0.4)  # a power of two: exact
    assert np.array_equal(i1, i4) and np.array_equal(C4, 4.0 * C1)


def test_w8_rejects_non_int8_weights():
    with pytest.raises(TypeError):
        O.dequantize_w8(np.zeros((2, 2), dtype=np.int16), np.ones(2))


# ---------------------------------------------------------------- P·V with its softmax producer
def test_round_bf16_matches_the_format():
    # halfway cases go to the even significand; exact values stay
    got = O.round_bf16(np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -7, 0.75, -(1 + 2 ** -8), 3 * 2 ** -130,
                                 2.0 ** 100 * (1 + 2 ** -9)]))
    want = np.array([1.0, 1.0, 1 + 2 ** -6, 1 + 2 ** -7, 0.75, -1.0, 3 * 2 ** -130, 2.0 ** 100])
    assert np.array_equal(got, want)
    # and a library routine that implements the same rounding (torch's float64 -> bfloat16 cast)
    import torch
    r = np.random.default_rng(3)
    x = r.standard_normal(20000) * np.exp(4 * r.standard_normal(20000))
    assert np.array_equal(O.round_bf16(x), torch.tensor(x).to(torch.bfloat16).double().numpy())


def test_causal_softmax_hand_example():
    L = np.array([[0.0, 5.0, 7.0], [np.log(2.0), 0.0, 9.0], [0.0, np.log(3.0), 0.0]])
    P = O.causal_softmax(L)
    want = np.array([[1.0, 0.0, 0.0], [2 / 3, 1 / 3, 0.0], [0.2, 0.6, 0.2]])
    assert np.allclose(P, want, rtol=0, atol=1e-15)
    assert P[0, 1] == 0.0 and P[0, 2] == 0.0 and P[1, 2] == 0.0  # masked entries exactly zero
    # without the mask every key counts
    Pn = O.causal_softmax(L, causal=False)
    assert np.allclose(Pn[0], np.exp([0.0, 5.0, 7.0]) / np.exp([0.0, 5.0, 7.0]).sum(), rtol=1e-14)
    # fewer queries than keys: the last query sees every key, the mask is aligned to it
    P2 = O.causal_softmax(np.zeros((2, 3)))
    assert np.allclose(P2, [[0.5, 0.5, 0.0], [1 / 3, 1 / 3, 1 / 3]], rtol=0, atol=1e-15)


def test_causal_softmax_invariants():
    r = np.random.default_rng(11)
    L = 3.0 * r.standard_normal((2, 9, 9))
    P = O.causal_softmax(L)
    assert np.allclose(P.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(P[:, np.triu_indices(9, 1)[0], np.triu_indices(9, 1)[1]] == 0.0)
    # a constant added to each row changes nothing; a zero scale gives the uniform distribution
    assert np.allclose(O.causal_softmax(L + r.standard_normal((2, 9, 1))), P, rtol=1e-12, atol=1e-15)
    U = O.causal_softmax(L, scale=0.0)
    assert np.allclose(U[0, 4, :5], 0.2, rtol=0, atol=1e-15)
    # the scale multiplies the logits
    assert np.allclose(O.causal_softmax(L, scale=0.5), O.causal_softmax(0.5 * L), rtol=1e-14, atol=0)


def test_pv_softmax_pipeline_stores_bf16_and_reduces_over_keys():
    r = np.random.default_rng(12)
    L = 3.0 * r.standard_normal((2, 12, 12))
    V = r.standard_normal((2, 12, 4))
    O_, idx, s, P = O.pv_softmax_reduced(L, V, 1.0)
    # P is the bf16 rounding of the softmax, and rho = 1 is the whole product P·V
    assert np.array_equal(P, O.round_bf16(O.causal_softmax(L)))
    assert np.allclose(O_, P @ V, rtol=1e-13, atol=1e-15)
    # the causal mask makes the last key's column the sparsest: only the last query sees it
    assert np.count_nonzero(P[:, :, -1]) == 2
    O5, idx5, s5, _ = O.pv_softmax_reduced(L, V, 0.5)
    assert idx5.shape == (2, 6)
