"""fp64 CPU oracle for Reduced Matrix Multiplication (RMM).

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this module. It shares no code with the
CUDA library: it is a plain NumPy restatement of the method, in float64, written
so that each step can be checked against the pages by eye.

Sources (web pages on the paper "Reduced Matrix Multiplication: Input-Adaptive
Matrix-Product Reduction for LLM Inference"):

* gist.science, Portuguese summary, "Resumo Técnico" › "Metodologia":
  - "Mecanismo Central": pick a subset I of the shared contraction dimension d
    and compute the reduced product A[:, I] · B[I, :] instead of A · B.
  - "Estratégia de Seleção": score feature j by the column norm ‖A[:, j]‖₂ of
    the activation matrix and keep the top-k indices, k = ⌈ρ·d⌉, ρ the
    user-controlled retention ratio.
  - "Base Teórica": top-k by column norm is minimax-optimal for the worst-case
    approximation error over all weight matrices B when only A is known.
* shd-paper.top, abstract: RMM selects informative slices along the contraction
  dimension of each matrix product, without modifying the weights.

Readings taken where the pages are silent (each is a library default too):

* The default slice score multiplies the activation column norm by the norm of
  the matching row of B: s_k = ‖A[:, k]‖₂ · ‖B[k, :]‖₂ ("product" mode). The
  pages' own activation-only score ‖A[:, k]‖₂ is the "a_only" mode.
* Ties in the score are broken toward the lower index; the kept indices are
  returned in ascending order.
* k = ⌈ρ·K⌉ is evaluated as the ceiling of the IEEE double product ρ·K, with ρ
  restricted to (0, 1].
* One selection per matrix product: every row of A uses the same index set. In
  a batch (attention heads) each batch item has its own selection.
* A non-finite score makes the result undefined; the oracle reports it.

Parity pins (tests/test_oracle_pins.py): hand-worked examples with closed-form
values (tests/golden/), exact integer arithmetic for ρ = 1 and for the split
A·B = A_S·B_S + A_D·B_D, the triangle-inequality error bound, brute force over
every subset on tiny inputs, the B = I closed form, zero slices ranked last,
and the minimax statement checked by construction. The softmax producer of
P·V: a hand-worked causal softmax, row sums, shift and scale invariants, and
the bf16 rounding against hand-picked halfway cases and torch's own cast.
"""
from __future__ import annotations

import math

import numpy as np

SCORE_PRODUCT = "product"
SCORE_A_ONLY = "a_only"


def keep_count(rho: float, K: int) -> int:
    """Number of kept slices k = ⌈ρ·K⌉ ("Estratégia de Seleção").

    ρ must lie in (0, 1] and K must be at least 1; the product ρ·K is the IEEE
    double product, as the library computes it."""
    if not (0.0 < rho <= 1.0) or K < 1:
        raise ValueError(f"keep_count: need 0 < rho <= 1 and K >= 1, got rho={rho}, K={K}")
    return int(math.ceil(rho * K))


def column_norms(A: np.ndarray) -> np.ndarray:
    """‖A[:, k]‖₂ for every column k of A (M×K), in float64."""
    A = np.asarray(A, dtype=np.float64)
    return np.sqrt(np.sum(A * A, axis=0))


def row_norms(B: np.ndarray) -> np.ndarray:
    """‖B[k, :]‖₂ for every row k of B (K×N), in float64."""
    B = np.asarray(B, dtype=np.float64)
    return np.sqrt(np.sum(B * B, axis=1))


def slice_scores(A: np.ndarray, B: np.ndarray, mode: str = SCORE_PRODUCT) -> np.ndarray:
    """Importance score of every contraction slice k of the product A·B.

    a_only:  s_k = ‖A[:, k]‖₂                    (the pages' activation column norm)
    product: s_k = ‖A[:, k]‖₂ · ‖B[k, :]‖₂        (the library's default)
    """
    a = column_norms(A)
    if mode == SCORE_A_ONLY:
        return a
    if mode != SCORE_PRODUCT:
        raise ValueError(f"unknown score mode {mode!r}")
    if B.shape[0] != A.shape[1]:
        raise ValueError("A and B disagree on the contraction dimension")
    return a * row_norms(B)


def select_top(s: np.ndarray, k_keep: int) -> np.ndarray:
    """Indices of the k_keep largest scores, ties toward the lower index,
    returned in ascending order ("Estratégia de Seleção": keep the top-k)."""
    s = np.asarray(s, dtype=np.float64)
    if not np.all(np.isfinite(s)):
        raise FloatingPointError("non-finite slice score")
    if not (1 <= k_keep <= s.shape[0]):
        raise ValueError(f"k_keep={k_keep} outside [1, {s.shape[0]}]")
    # A stable sort of -s keeps equal scores in index order, so among equal
    # scores the lower index comes first.
    order = np.argsort(-s, kind="stable")
    return np.sort(order[:k_keep]).astype(np.int64)


def pack(A: np.ndarray, B: np.ndarray, idx: np.ndarray):
    """A_S = A[:, I] (M×k) and B_S = B[I, :] (k×N) ("Mecanismo Central").

    I is a subset of the contraction indices {0, …, K−1}: an index outside
    that range is an error here (NumPy would wrap a negative one around)."""
    idx = np.asarray(idx)
    K = A.shape[1]
    if idx.size and (idx.min() < 0 or idx.max() >= K):
        raise IndexError(f"kept index outside [0, {K})")
    return A[:, idx], B[idx, :]


def reduced_product(A: np.ndarray, B: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """A[:, I] · B[I, :] in float64 ("Mecanismo Central")."""
    A_S, B_S = pack(np.asarray(A, dtype=np.float64), np.asarray(B, dtype=np.float64), idx)
    return A_S @ B_S


def matmul_reduced(A: np.ndarray, B: np.ndarray, rho: float, mode: str = SCORE_PRODUCT):
    """The whole method on one product: score → top-⌈ρK⌉ → reduced product.

    Returns (C, idx, s)."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    s = slice_scores(A, B, mode)
    idx = select_top(s, keep_count(rho, A.shape[1]))
    return reduced_product(A, B, idx), idx, s


def matmul_reduced_batched(A: np.ndarray, B: np.ndarray, rho: float, mode: str = SCORE_PRODUCT):
    """One independent selection per batch item: A [b][M][K], B [b][K][N]."""
    Cs, idxs, ss = [], [], []
    for b in range(A.shape[0]):
        C, idx, s = matmul_reduced(A[b], B[b], rho, mode)
        Cs.append(C)
        idxs.append(idx)
        ss.append(s)
    return np.stack(Cs), np.stack(idxs), np.stack(ss)


def qk_reduced(Q: np.ndarray, Kmat: np.ndarray, rho: float, mode: str = SCORE_PRODUCT):
    """Q·Kᵀ per head, reduced over the head dimension ("Escopo de Aplicação").

    Q [bh][S_q][d], Kmat [bh][S_k][d]; the contraction slices are head-dim
    channels, so B = Kᵀ and row k of B is column k of Kmat."""
    return matmul_reduced_batched(Q, np.swapaxes(Kmat, 1, 2), rho, mode)


def pv_reduced(P: np.ndarray, V: np.ndarray, rho: float, mode: str = SCORE_PRODUCT):
    """P·V per head, reduced over the key (token) dimension ("Escopo de Aplicação").

    P [bh][S_q][S_k], V [bh][S_k][d]."""
    return matmul_reduced_batched(P, V, rho, mode)


def dequantize_w8(Wq: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """INT8 weight with one scale per output channel ("Resultados
    Experimentais" › "Compatibilidade": the method works with INT8 weight
    quantization; the scheme is not given, so the plainest symmetric
    per-column form is read): W[k, n] = Wq[k, n] · scale[n], Wq in [-127, 127]."""
    Wq = np.asarray(Wq)
    if Wq.dtype != np.int8:
        raise TypeError("Wq must be int8")
    return Wq.astype(np.float64) * np.asarray(scale, dtype=np.float64)[None, :]


def matmul_reduced_w8(A: np.ndarray, Wq: np.ndarray, scale: np.ndarray, rho: float, mode: str = SCORE_PRODUCT):
    """RMM on an INT8 weight: the method applied to the dequantized weight, so
    the score is ‖A[:, k]‖₂ · ‖W[k, :]‖₂ of the dequantized W and the product
    is A[:, I] · W[I, :]. Returns (C, idx, s)."""
    return matmul_reduced(A, dequantize_w8(Wq, scale), rho, mode)


def frobenius_rel_error(C_test: np.ndarray, C_ref: np.ndarray) -> float:
    """‖C_test − C_ref‖_F / ‖C_ref‖_F (0 when both are zero)."""
    C_test = np.asarray(C_test, dtype=np.float64)
    C_ref = np.asarray(C_ref, dtype=np.float64)
    den = np.linalg.norm(C_ref)
    num = np.linalg.norm(C_test - C_ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else math.inf
    return float(num / den)


def selection_matches(gpu_idx: np.ndarray, oracle_idx: np.ndarray, s: np.ndarray,
                      rel_window: float = 1e-5):
    """Compare a computed kept-index set with the oracle's.

    Returns (ok, n_boundary): ok is True when every index in the symmetric
    difference of the two sets has an oracle score within rel_window·t of t, the
    oracle's k-th largest score (a near-tie at the selection boundary, where
    either choice is correct); n_boundary counts those indices. A computed set
    with an index outside [0, K) or a repeated index never matches."""
    s = np.asarray(s, dtype=np.float64)
    g_list = [int(i) for i in np.asarray(gpu_idx).ravel()]
    # I is a set of contraction indices: each in [0, K), none repeated
    if any(i < 0 or i >= s.shape[0] for i in g_list) or len(set(g_list)) != len(g_list):
        return False, 0
    g = set(g_list)
    o = set(int(i) for i in np.asarray(oracle_idx).ravel())
    if len(g) != len(o):
        return False, 0
    diff = g ^ o
    if not diff:
        return True, 0
    t = float(np.min(s[list(o)]))
    ok = all(abs(s[k] - t) <= rel_window * t for k in diff)
    return ok, len(diff)


# ---------------------------------------------------------------- P·V with its softmax producer
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties
    to even: the stored P of the attention workload. Written from the format's
    definition (value = significand · 2^e with an 8-bit significand), not from
    any library routine. Finite inputs of normal bf16 range only."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    # exact powers of two can land one off in log2; fix the exponent so that
    # |x| / 2^e lies in [1, 2)
    m = np.abs(x[nz]) / np.exp2(e)
    e = np.where(m >= 2.0, e + 1, np.where(m < 1.0, e - 1, e))
    q = x[nz] / np.exp2(e - 7)          # significand scaled to an integer grid of 2^7 steps
    out[nz] = np.rint(q) * np.exp2(e - 7)  # np.rint rounds halves to even
    return out


def causal_softmax(L: np.ndarray, scale: float = 1.0, causal: bool = True) -> np.ndarray:
    """Row softmax of scale·L in float64 ("Escopo de Aplicação": P is the
    attention matrix, P = softmax of the scaled logits). With the causal mask,
    query row q sees key k only when k <= q + (S_k - S_q) (the last query sees
    every key); masked entries of P are 0. L: [..., S_q, S_k]."""
    L = np.asarray(L, dtype=np.float64) * scale
    S_q, S_k = L.shape[-2], L.shape[-1]
    if causal:
        q = np.arange(S_q)[:, None]
        k = np.arange(S_k)[None, :]
        visible = k <= q + (S_k - S_q)
        L = np.where(visible, L, -np.inf)
    m = np.max(L, axis=-1, keepdims=True)
    E = np.exp(L - m)
    return E / np.sum(E, axis=-1, keepdims=True)


def pv_softmax_reduced(L: np.ndarray, V: np.ndarray, rho: float, mode: str = SCORE_PRODUCT, scale: float = 1.0,
                       causal: bool = True):
    """P·V with P produced from the logits, in the pages' order: P = softmax
    (stored as bf16), the slice scores of P·V, the top-ceil(rho·S_k) keys per
    head, the reduced product over them ("Escopo de Aplicação": P·V reduced
    over the keys). L [bh][S_q][S_k], V [bh][S_k][d]. Returns (O, idx, s, P)
    with P the stored bf16 values as float64."""
    P = round_bf16(causal_softmax(L, scale, causal))
    O, idx, s = pv_reduced(P, np.asarray(V, dtype=np.float64), rho, mode)
    return O, idx, s, P
