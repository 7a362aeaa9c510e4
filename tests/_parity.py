"""Shared parity helpers: run the library (through the C ABI) and the fp64
oracle on the same inputs and compare them under the stated rules:

* slice scores: relative error <= 1e-5 against the fp64 scores;
* kept index set: every index in [0, K), strictly ascending, and identical to
  the oracle's, except indices whose oracle score lies within 1e-5·t of t, the
  k-th largest score (near-ties at the boundary, where either choice is
  correct);
* product, against the oracle's product over the library's own kept set:
  - relative Frobenius error <= 1e-2 when bf16 is involved and <= 1e-5 for
    f32 inputs with f32 output (the stated tolerance), and
  - element by element, a forward-error bound of f32 accumulation (below), so
    that a fault confined to a few entries (one wrong tile, a missing split-K
    partial sum, a bad column) cannot hide inside a whole-matrix norm.

Element-wise bound. Let y = sum_t a_t b_t over the k kept slices (exact, fp64
oracle) and S = sum_t |a_t| |b_t| (the entry of |A_S|·|B_S|). The library
forms every product exactly in f32 (bf16 x bf16, and bf16 x int8, fit in 24
significant bits; f32 x f32 products are fused into the FMA) and adds the k
products in f32 along some tree whose height is at most K + 16, K the full
contraction length (tensor-core K-groups, split-K reduce-adds, cluster
partial sums; the route that streams A whole adds the dropped slices as
exact zeros). Each addition errs by at most 2u relative (u = 2^-24; the
factor 2 admits accumulators that truncate instead of rounding to nearest),
so the f32 result obeys
    |y_f32 - y| <= E = g·S,   g = 2u·(K + 16) / (1 - 2u·(K + 16)).
A final scaling (the INT8 column scale) and the store add at most
2u·(|y| + E); rounding the result to bf16 adds at most 2^-8·(|y| + E) (bf16
has 8 significant bits, round to nearest even); weights rounded to bf16
before the product (the INT8 pack route) add at most 2^-8·S.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import rmm_oracle as O

SCORE_RTOL = 1e-5
WINDOW = 1e-5
U_F32 = 2.0 ** -24   # unit roundoff of f32 (24 significant bits, round to nearest)
U_BF16 = 2.0 ** -8   # unit roundoff of bf16 (8 significant bits, round to nearest even)
ACC_FACTOR = 2.0     # per-addition error in units of U_F32 (truncating accumulation allowed)
TREE_SLACK = 16      # extra levels of the summation tree beyond K


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16/f32 tensor on the host."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def product_tol(in_dtype, out_dtype) -> float:
    return 1e-5 if (in_dtype == torch.float32 and out_dtype == torch.float32) else 1e-2


def check_scores(s_gpu: np.ndarray, s_ref: np.ndarray):
    s_gpu = np.asarray(s_gpu, dtype=np.float64)
    zero = s_ref == 0
    assert np.all(s_gpu[zero] == 0), "zero slice scored nonzero"
    nz = ~zero
    if np.any(nz):
        rel = np.abs(s_gpu[nz] - s_ref[nz]) / s_ref[nz]
        assert rel.max() <= SCORE_RTOL, f"score rel err {rel.max():.3e}"


def check_index_list(idx_gpu: np.ndarray, K: int, k_keep: int | None = None) -> np.ndarray:
    """The kept indices as int64, after checking that there are k_keep of them,
    each in [0, K), strictly ascending (a negative index would otherwise wrap
    around in NumPy indexing)."""
    idx = np.asarray(idx_gpu).astype(np.int64).ravel()
    if k_keep is not None:
        assert idx.shape == (k_keep,), f"{idx.shape[0]} kept indices, expected {k_keep}"
    assert idx.size == 0 or (idx.min() >= 0 and idx.max() < K), \
        f"kept index outside [0, {K}): min {idx.min()}, max {idx.max()}"
    assert np.all(np.diff(idx) > 0), "kept indices not strictly ascending"
    return idx


def check_selection(idx_gpu: np.ndarray, s_ref: np.ndarray, k_keep: int) -> int:
    idx = check_index_list(idx_gpu, s_ref.shape[0], k_keep)
    o = O.select_top(s_ref, k_keep)
    ok, n = O.selection_matches(idx, o, s_ref, WINDOW)
    assert ok, f"selection differs outside the near-tie window ({n} indices differ)"
    return n


def element_bound(A_S: np.ndarray, B_S: np.ndarray, ref: np.ndarray, out_bf16: bool, w_rel: float = 0.0,
                  K: int | None = None):
    """Largest admissible |C - ref| per entry for the f32-accumulated product
    of the kept operands A_S (M x k) and B_S (k x N) out of K slices; see the
    module docstring."""
    K = A_S.shape[1] if K is None else K
    S = np.abs(A_S) @ np.abs(B_S)
    h = ACC_FACTOR * U_F32 * (K + TREE_SLACK)
    E = (h / (1.0 - h)) * S
    mag = np.abs(ref) + E
    bound = E + 2.0 * U_F32 * mag + w_rel * S
    if out_bf16:
        bound = bound + U_BF16 * mag
    return bound


def check_product(C_gpu, A64: np.ndarray, B64: np.ndarray, idx: np.ndarray, tol: float, *,
                  out_dtype: torch.dtype | None = None, w_rel: float = 0.0):
    """Compare C with the oracle's product over the kept set idx: the relative
    Frobenius tolerance `tol` and the per-entry forward-error bound.

    C_gpu is the library's output as a tensor (its dtype decides whether the
    bf16 output rounding enters the bound) or as an array, in which case
    out_dtype must be given. w_rel: relative rounding of B's values before the
    product (2^-8 when INT8 weights are converted to bf16 for the GEMM)."""
    if isinstance(C_gpu, torch.Tensor):
        out_dtype = C_gpu.dtype
        C_gpu = f64(C_gpu)
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("check_product needs the output dtype (pass the tensor or out_dtype=)")
    A64 = np.asarray(A64, dtype=np.float64)
    B64 = np.asarray(B64, dtype=np.float64)
    I = check_index_list(idx, A64.shape[1])
    assert B64.shape[0] == A64.shape[1], "A and B disagree on the contraction dimension"
    C_gpu = np.asarray(C_gpu, dtype=np.float64)
    ref = O.reduced_product(A64, B64, I)
    assert C_gpu.shape == ref.shape, f"product shape {C_gpu.shape}, expected {ref.shape}"
    assert np.all(np.isfinite(C_gpu)), "non-finite product entries"
    err = O.frobenius_rel_error(C_gpu, ref)
    assert err <= tol, f"product rel Frobenius error {err:.3e} > {tol}"
    bound = element_bound(A64[:, I], B64[I, :], ref, out_dtype == torch.bfloat16, w_rel, K=A64.shape[1])
    excess = np.abs(C_gpu - ref) - bound
    if np.any(excess > 0):
        i, j = np.unravel_index(int(np.argmax(excess)), excess.shape)
        n_bad = int(np.count_nonzero(excess > 0))
        raise AssertionError(
            f"{n_bad} product entries outside the f32 forward-error bound; worst at ({i}, {j}): "
            f"got {C_gpu[i, j]:.9g}, oracle {ref[i, j]:.9g}, bound {bound[i, j]:.3g}")
    return err


def check_single(A: torch.Tensor, B: torch.Tensor, rho: float, mode: str, C: torch.Tensor, idx: torch.Tensor,
                 b_kmajor: bool = False):
    """End-to-end check of one (unbatched) product."""
    A64 = f64(A)
    B64 = f64(B).T if b_kmajor else f64(B)
    k = O.keep_count(rho, A64.shape[1])
    s_ref = O.slice_scores(A64, B64, mode)
    n_boundary = check_selection(idx.cpu().numpy(), s_ref, k)
    err = check_product(C, A64, B64, idx.cpu().numpy(), product_tol(A.dtype, C.dtype))
    return n_boundary, err
