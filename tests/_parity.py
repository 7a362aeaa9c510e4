"""Shared parity helpers: run the library (through the C ABI) and the fp64
oracle on the same inputs and compare them under the stated rules:

* slice scores: relative error <= 1e-5 against the fp64 scores;
* kept index set: identical to the oracle's, except indices whose oracle score
  lies within 1e-5·t of t, the k-th largest score (near-ties at the boundary,
  where either choice is correct);
* product: relative Frobenius error, against the oracle's product over the
  library's own kept set, <= 1e-2 when bf16 is involved and <= 1e-5 for f32
  inputs with f32 output.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import rmm_oracle as O

SCORE_RTOL = 1e-5
WINDOW = 1e-5


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


def check_selection(idx_gpu: np.ndarray, s_ref: np.ndarray, k_keep: int) -> int:
    idx_gpu = np.asarray(idx_gpu).astype(np.int64)
    assert idx_gpu.shape == (k_keep,)
    assert np.all(np.diff(idx_gpu) > 0), "kept indices not strictly ascending"
    o = O.select_top(s_ref, k_keep)
    ok, n = O.selection_matches(idx_gpu, o, s_ref, WINDOW)
    assert ok, f"selection differs outside the near-tie window ({n} indices differ)"
    return n


def check_product(C_gpu: np.ndarray, A64: np.ndarray, B64: np.ndarray, idx: np.ndarray, tol: float):
    ref = O.reduced_product(A64, B64, np.asarray(idx).astype(np.int64))
    err = O.frobenius_rel_error(C_gpu, ref)
    assert err <= tol, f"product rel Frobenius error {err:.3e} > {tol}"
    return err


def check_single(A: torch.Tensor, B: torch.Tensor, rho: float, mode: str, C: torch.Tensor, idx: torch.Tensor,
                 b_kmajor: bool = False):
    """End-to-end check of one (unbatched) product."""
    A64 = f64(A)
    B64 = f64(B).T if b_kmajor else f64(B)
    k = O.keep_count(rho, A64.shape[1])
    s_ref = O.slice_scores(A64, B64, mode)
    n_boundary = check_selection(idx.cpu().numpy(), s_ref, k)
    err = check_product(f64(C), A64, B64, idx.cpu().numpy(), product_tol(A.dtype, C.dtype))
    return n_boundary, err
