"""Python binding for librmm, the B200 Reduced Matrix Multiplication library.

Argument marshalling only: every step of score -> select -> pack -> gemm runs in
the library's CUDA kernels. PyTorch supplies device memory and the current
stream. There is no fallback: if librmm.so is missing, loading fails loudly.

Method (gist.science summary of "Reduced Matrix Multiplication: Input-Adaptive
Matrix-Product Reduction for LLM Inference", Resumo Técnico › Metodologia):
score every contraction slice k of A·B, keep the top ceil(rho·K), and compute
A[:, I]·B[I, :]. The default score is ||A[:,k]||·||B[k,:]|| ("product"); the
pages' activation-only column norm is mode "a_only".
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librmm.so")

RMM_OK, RMM_ERR_INVALID, RMM_ERR_NONFINITE, RMM_ERR_CUDA, RMM_ERR_TIMEOUT, RMM_ERR_UNSUPPORTED = range(6)
RMM_BF16, RMM_F32 = 0, 1
SCORE_MODES = {"product": 0, "a_only": 1}
STATUS_NAMES = {0: "RMM_OK", 1: "RMM_ERR_INVALID", 2: "RMM_ERR_NONFINITE", 3: "RMM_ERR_CUDA",
                4: "RMM_ERR_TIMEOUT", 5: "RMM_ERR_UNSUPPORTED"}


class RMMError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None

_vp, _i64, _f64, _i32, _u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_uint64
_SIGS = {
    "rmm_keep_count": (_i64, [_f64, _i64]),
    "rmm_padded_keep": (_i64, [_i64]),
    "rmm_packed_b_ld": (_i64, [_i64]),
    "rmm_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _i64, _i32]),
    "rmm_workspace_size_for": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _i64, _i32, _i32]),
    "rmm_score": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i32, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _vp,
                         _vp]),
    "rmm_select": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "rmm_pack": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i32, _i64, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _vp,
                        _vp, _vp]),
    "rmm_gemm": (_i32, [_vp, _vp, _i32, _i64, _i64, _i64, _i64, _i32, _vp, _i64, _i64, _i32, _vp, _vp]),
    "rmm_matmul_reduced": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _i64, _f64, _i32, _i32, _vp, _i64, _i32, _vp,
                                  _vp, ctypes.c_size_t, _vp]),
    "rmm_matmul_reduced_batched": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i32, _i64, _i64, _i64, _i64, _f64,
                                          _i32, _i32, _vp, _i64, _i64, _i32, _vp, _vp, ctypes.c_size_t, _vp]),
    "rmm_qk_reduced": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _f64, _i32, _i32, _vp, _i32, _vp, _vp,
                              ctypes.c_size_t, _vp]),
    "rmm_pv_reduced": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _f64, _i32, _i32, _vp, _i32, _vp, _vp,
                              ctypes.c_size_t, _vp]),
    "rmm_matmul_reduced_noalloc": (_i32, [_vp, _i64, _vp, _i64, _i64, _i64, _i64, _f64, _i32, _i32, _vp, _i64, _i32,
                                          _vp, _vp, _vp]),
    "rmm_b_norms": (_i32, [_vp, _i64, _i64, _i32, _i64, _i64, _i64, _i32, _vp, _vp, _vp]),
    "rmm_score_b_norms": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _i32, _vp, _vp, _vp]),
    "rmm_matmul_reduced_b_norms": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i32, _vp, _i64, _i64, _i64, _i64,
                                          _i64, _f64, _i32, _vp, _i64, _i64, _i32, _vp, _vp, ctypes.c_size_t,
                                          _vp]),
    "rmm_gemv_gather": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _vp, _i64, _i32, _vp,
                               _i64, _i64, _i32, _vp]),
    "rmm_b_norms_w8": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _vp]),
    "rmm_pack_w8": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _i64, _vp,
                           _vp, _vp, _vp]),
    "rmm_matmul_reduced_w8": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _i64, _i64, _i64,
                                     _i64, _f64, _i32, _i32, _vp, _i64, _i64, _i32, _vp, _vp, ctypes.c_size_t,
                                     _vp]),
    "rmm_gemv_gather_w8": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _i64,
                                  _vp, _i64, _i64, _i32, _vp]),
    "rmm_mask_rows": (_i32, [_vp, _i64, _i64, _i64, _i64, _i64, _vp, _i64, _i32, _vp, _vp]),
    "rmm_gemm_full": (_i32, [_vp, _i64, _i64, _vp, _i64, _i64, _i64, _i64, _i64, _i32, _vp, _i64, _i64, _i32, _vp,
                             _vp]),
    "rmm_fused_route": (_i32, [_i64, _i64, _i64, _i32, _i32, _vp, _i64, _i64]),
    "rmm_softmax_row_stats": (_i32, [_vp, _i32, ctypes.c_float, _i32, _i64, _i64, _i64, _vp, _vp, _vp]),
    "rmm_softmax_score": (_i32, [_vp, _i32, ctypes.c_float, _i32, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _vp,
                                 _vp]),
    "rmm_pv_softmax_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64, _i64]),
    "rmm_pv_softmax_reduced": (_i32, [_vp, _i32, ctypes.c_float, _i32, _vp, _i64, _i64, _i64, _i64, _f64, _i32, _vp,
                                      _vp, _i32, _vp, _vp, ctypes.c_size_t, _vp]),
    "rmm_check": (_i32, [_vp, _vp]),
    "rmm_last_error_string": (ctypes.c_char_p, []),
    "rmm_set_wait_limit_ns": (None, [_u64]),
    "rmm_set_stall_producer_for_test": (None, [_i32]),
    "rmm_set_gemm_cta_group": (_i32, [_i32]),
    "rmm_launch_count": (_u64, []),
    "rmm_set_debug": (_i32, [_i32]),
    "rmm_set_gemm_events": (None, [ctypes.c_void_p, ctypes.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """The loaded librmm.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"librmm.so not found at {_LIB_PATH}; build it with "
                              "`python -m input_adaptive_reduced_02_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def library_path() -> str:
    return _LIB_PATH


def _check(status: int):
    if status != RMM_OK:
        raise RMMError(status, lib().rmm_last_error_string().decode(errors="replace"))


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RMM_BF16
    if t.dtype == torch.float32:
        return RMM_F32
    raise TypeError(f"unsupported dtype {t.dtype}; librmm takes bfloat16 or float32")


def _out_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return RMM_BF16
    if dt == torch.float32:
        return RMM_F32
    raise TypeError(f"unsupported output dtype {dt}")


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _mat(t: torch.Tensor, name: str):
    """(batch, rows, cols, ld, batch_stride) of a 2-D or 3-D CUDA tensor."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() == 2:
        t3 = t.unsqueeze(0)
    elif t.dim() == 3:
        t3 = t
    else:
        raise ValueError(f"{name} must be 2-D or 3-D")
    if t3.stride(2) != 1 and t3.shape[2] > 1:
        raise ValueError(f"{name} must be contiguous along its last dimension")
    b, r, c = t3.shape
    ld = t3.stride(1) if r > 1 else c
    bs = t3.stride(0) if b > 1 else r * ld
    return b, r, c, ld, bs


def keep_count(rho: float, K: int) -> int:
    k = lib().rmm_keep_count(float(rho), int(K))
    if k < 1:
        raise ValueError(f"rho must lie in (0, 1] and K >= 1 (rho={rho}, K={K})")
    return int(k)


def padded_keep(k_keep: int) -> int:
    return int(lib().rmm_padded_keep(int(k_keep)))


def workspace_size(batch: int, M: int, K: int, N: int, k_keep: int, dtype: torch.dtype) -> int:
    """Workspace bytes of a fused call on any route."""
    return int(lib().rmm_workspace_size(batch, M, K, N, k_keep, _out_code(dtype)))


def workspace_size_for(batch: int, M: int, K: int, N: int, k_keep: int, dtype: torch.dtype,
                       b_kmajor: bool = False) -> int:
    """Workspace bytes of a fused call on the route it takes (no packed operands when M <= 16 and B is row-major)."""
    return int(lib().rmm_workspace_size_for(batch, M, K, N, k_keep, _out_code(dtype), int(b_kmajor)))


class Workspace:
    """A 1 KiB-aligned device workspace carved from one torch allocation."""

    def __init__(self, nbytes: int, device):
        self.nbytes = int(nbytes)
        self._buf = torch.empty(self.nbytes + 1024, dtype=torch.uint8, device=device)
        base = self._buf.data_ptr()
        self.offset = (-base) % 1024
        self.ptr = base + self.offset

    @property
    def status_ptr(self) -> int:
        return self.ptr


def _ensure_ws(ws, nbytes, device):
    if ws is None or ws.nbytes < nbytes:
        return Workspace(nbytes, device)
    return ws


def status_word(device="cuda") -> torch.Tensor:
    """A zeroed device u32 (as int32 storage) for the stage calls' status bits."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def check(status, stream_tensor: torch.Tensor | None = None):
    """Read and clear a device status word (a tensor from status_word(), or a
    Workspace); raise RMMError on NaN/Inf scores or a pipeline timeout."""
    if isinstance(status, Workspace):
        ptr, dev = status.ptr, status._buf.device
    else:
        ptr, dev = status.data_ptr(), status.device
    st = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    _check(lib().rmm_check(ctypes.c_void_p(ptr), st))


# ---------------------------------------------------------------- stage calls
def score(A: torch.Tensor, B: torch.Tensor | None, mode: str = "product", b_kmajor: bool = False,
          out: torch.Tensor | None = None, status: torch.Tensor | None = None) -> torch.Tensor:
    """Slice scores s [batch][K] (f32). A [b][M][K]; B [b][K][N] (or [b][N][K] with b_kmajor)."""
    ba, M, K, lda, sA = _mat(A, "A")
    if B is not None:
        bb, r, c, ldb, sB = _mat(B, "B")
        N = r if b_kmajor else c
        if (c if b_kmajor else r) != K or bb != ba:
            raise ValueError("A and B disagree on the contraction dimension or batch")
    else:
        if SCORE_MODES[mode] != 1:
            raise ValueError("B is required in product mode")
        N, ldb, sB = 0, 0, 0
    if out is None:
        out = torch.empty((ba, K) if A.dim() == 3 else (K,), dtype=torch.float32, device=A.device)
    _check(lib().rmm_score(_ptr(A), lda, sA, _ptr(B), ldb, sB, int(b_kmajor), ba, M, K, N, _dtype(A),
                           SCORE_MODES[mode], _ptr(out), _ptr(status), _stream(A)))
    return out


def b_norms(B: torch.Tensor, b_kmajor: bool = False, out: torch.Tensor | None = None,
            status: torch.Tensor | None = None) -> torch.Tensor:
    """B's factor of the product score, ||B[k,:]||_2 per slice k (f32 [batch][K] or [K]),
    for reuse across calls while B is unchanged. B [b][K][N] (or Kmat [b][N][K] with b_kmajor)."""
    bb, r, c, ldb, sB = _mat(B, "B")
    K, N = (c, r) if b_kmajor else (r, c)
    if out is None:
        out = torch.empty((bb, K) if B.dim() == 3 else (K,), dtype=torch.float32, device=B.device)
    _check(lib().rmm_b_norms(_ptr(B), ldb, sB, int(b_kmajor), bb, K, N, _dtype(B), _ptr(out), _ptr(status),
                             _stream(B)))
    return out


def _bn_stride(b_norm: torch.Tensor, batch: int, K: int) -> int:
    if b_norm.dtype != torch.float32 or not b_norm.is_cuda or not b_norm.is_contiguous():
        raise ValueError("b_norm must be a contiguous float32 CUDA tensor")
    if b_norm.dim() == 1:
        if b_norm.shape[0] != K:
            raise ValueError("b_norm must hold K values")
        return 0  # one vector shared by every batch item
    if tuple(b_norm.shape) != (batch, K):
        raise ValueError("b_norm must be [K] or [batch][K]")
    return K


def score_b_norms(A: torch.Tensor, b_norm: torch.Tensor, out: torch.Tensor | None = None,
                  status: torch.Tensor | None = None) -> torch.Tensor:
    """Product-form slice scores with B's norms given: s[k] = ||A[:,k]||_2 · b_norm[k]."""
    ba, M, K, lda, sA = _mat(A, "A")
    stride = _bn_stride(b_norm, ba, K)
    if out is None:
        out = torch.empty((ba, K) if A.dim() == 3 else (K,), dtype=torch.float32, device=A.device)
    _check(lib().rmm_score_b_norms(_ptr(A), lda, sA, _ptr(b_norm), stride, ba, M, K, _dtype(A), _ptr(out),
                                   _ptr(status), _stream(A)))
    return out


def select(s: torch.Tensor, k_keep: int, out: torch.Tensor | None = None,
           status: torch.Tensor | None = None) -> torch.Tensor:
    """Ascending int32 indices of the k_keep largest scores per row of s (ties -> lower index)."""
    if s.dtype != torch.float32 or not s.is_cuda or not s.is_contiguous():
        raise ValueError("s must be a contiguous float32 CUDA tensor")
    batch, K = (1, s.shape[0]) if s.dim() == 1 else s.shape
    if out is None:
        out = torch.empty((k_keep,) if s.dim() == 1 else (batch, k_keep), dtype=torch.int32, device=s.device)
    _check(lib().rmm_select(_ptr(s), batch, K, k_keep, _ptr(out), _ptr(status), _stream(s)))
    return out


def packed_b_ld(N: int) -> int:
    return int(lib().rmm_packed_b_ld(int(N)))


def packed_b_shape(batched: bool, batch: int, N: int, k_pad: int, b_kmajor: bool):
    """Shape of the packed B operand: [(b)][N][k_pad] (b_kmajor) or [(b)][k_pad][packed_b_ld(N)]."""
    shp = (N, k_pad) if b_kmajor else (k_pad, packed_b_ld(N))
    return (batch, *shp) if batched else shp


def pack(A: torch.Tensor, B: torch.Tensor, idx: torch.Tensor, b_kmajor: bool = False, out=None,
         status: torch.Tensor | None = None):
    """A_S [b][M][k_pad] (kept columns of A, zero padded) and the packed B
    operand: the kept rows of B ([b][k_pad][packed_b_ld(N)]) or, with b_kmajor,
    the kept columns of Kmat ([b][N][k_pad]). `out` may supply the pair."""
    ba, M, K, lda, sA = _mat(A, "A")
    bb, r, c, ldb, sB = _mat(B, "B")
    N = r if b_kmajor else c
    k_keep = idx.shape[-1]
    kp = padded_keep(k_keep)
    bshape = packed_b_shape(A.dim() == 3, ba, N, kp, b_kmajor)
    if out is None:
        A_S = torch.empty((ba, M, kp) if A.dim() == 3 else (M, kp), dtype=A.dtype, device=A.device)
        B_S = torch.empty(bshape, dtype=A.dtype, device=A.device)
    else:
        A_S, B_S = out
        if A_S.numel() != ba * M * kp or B_S.numel() != int(torch.tensor(bshape).prod()):
            raise ValueError("pack: output buffers have the wrong size")
    _check(lib().rmm_pack(_ptr(A), lda, sA, _ptr(B), ldb, sB, int(b_kmajor), ba, M, K, N, _ptr(idx), k_keep,
                          _dtype(A), _ptr(A_S), _ptr(B_S), _ptr(status), _stream(A)))
    return A_S, B_S


def gemm(A_S: torch.Tensor, B_S: torch.Tensor, k_keep: int, out_dtype=torch.float32, b_kmajor: bool = False,
         N: int | None = None, out: torch.Tensor | None = None, status: torch.Tensor | None = None) -> torch.Tensor:
    """C = A_S · B_S over the first k_keep (of k_pad) slices; B_S as written by pack()."""
    ba, M, kp, _, _ = _mat(A_S, "A_S")
    if b_kmajor:
        N = B_S.shape[-2]
    elif N is None:
        N = B_S.shape[-1]
    if out is None:
        out = torch.empty((ba, M, N) if A_S.dim() == 3 else (M, N), dtype=out_dtype, device=A_S.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_gemm(_ptr(A_S), _ptr(B_S), int(b_kmajor), ba, M, N, k_keep, _dtype(A_S), _ptr(out), ldc, sC,
                          _out_code(out.dtype), _ptr(status), _stream(A_S)))
    return out


def gemv_gather(A: torch.Tensor, B: torch.Tensor, idx: torch.Tensor, out_dtype=torch.float32,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """C = A[:, idx] · B[idx, :] straight from A (M <= 16 rows) and row-major B, no packing."""
    ba, M, K, lda, sA = _mat(A, "A")
    bb, r, N, ldb, sB = _mat(B, "B")
    if r != K or bb != ba:
        raise ValueError("A and B disagree on the contraction dimension or batch")
    k = idx.shape[-1]
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_gemv_gather(_ptr(A), lda, sA, _ptr(B), ldb, sB, ba, M, K, N, _ptr(idx), k, _dtype(A),
                                 _ptr(out), ldc, sC, _out_code(out.dtype), _stream(A)))
    return out


ROUTE_PACK, ROUTE_STREAM, ROUTE_GEMV = 0, 1, 2


def fused_route(A: torch.Tensor, N: int, b_kmajor: bool = False) -> int:
    """Route a fused call takes for A (2-D or 3-D) and N: ROUTE_PACK,
    ROUTE_STREAM (B's dropped rows zeroed, A streamed whole) or ROUTE_GEMV."""
    ba, M, K, lda, sA = _mat(A, "A")
    return int(lib().rmm_fused_route(ba, M, N, int(b_kmajor), _dtype(A), _ptr(A), lda, sA))


def _fused_ws_bytes(A: torch.Tensor, N: int, k: int, b_kmajor: bool) -> int:
    """Workspace of a fused call on the route it takes for this A."""
    ba, M, K, _, _ = _mat(A, "A")
    if fused_route(A, N, b_kmajor) == ROUTE_PACK:
        return workspace_size(ba, M, K, N, k, A.dtype)
    return workspace_size_for(ba, M, K, N, k, A.dtype, b_kmajor)


def mask_rows(B: torch.Tensor, idx: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """B_M = B with the rows outside idx zeroed: [(b)][K][packed_b_ld(N)]."""
    bb, K, N, ldb, sB = _mat(B, "B")
    k = idx.shape[-1]
    if out is None:
        shp = (K, packed_b_ld(N))
        out = torch.empty((bb, *shp) if B.dim() == 3 else shp, dtype=B.dtype, device=B.device)
    _check(lib().rmm_mask_rows(_ptr(B), ldb, sB, bb, K, N, _ptr(idx), k, _dtype(B), _ptr(out), _stream(B)))
    return out


def gemm_full(A: torch.Tensor, B_M: torch.Tensor, N: int, out_dtype=torch.float32, out: torch.Tensor | None = None,
              status: torch.Tensor | None = None, causal_off: int = -1) -> torch.Tensor:
    """C = A · B_M over all K slices (bf16 tensor cores), B_M as mask_rows writes it.
    causal_off >= 0 declares A[i][k] = 0 for k > i + causal_off (blocks above are skipped)."""
    ba, M, K, lda, sA = _mat(A, "A")
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_gemm_full(_ptr(A), lda, sA, _ptr(B_M), ba, M, K, N, int(causal_off), _dtype(A), _ptr(out), ldc,
                               sC, _out_code(out.dtype), _ptr(status), _stream(A)))
    return out


# ---------------------------------------------------------------- fused calls
def matmul_reduced(A: torch.Tensor, B: torch.Tensor, rho: float, mode: str = "product",
                   out_dtype=torch.float32, out: torch.Tensor | None = None, workspace: Workspace | None = None,
                   idx_out: torch.Tensor | None = None, b_kmajor: bool = False):
    """C ≈ A·B keeping the top ceil(rho·K) contraction slices (batched when A is 3-D).

    Returns (C, workspace); the workspace can be passed back in to avoid
    re-allocation and to read the device status with check(workspace)."""
    ba, M, K, lda, sA = _mat(A, "A")
    bb, r, c, ldb, sB = _mat(B, "B")
    N = r if b_kmajor else c
    k = keep_count(rho, K)
    ws = _ensure_ws(workspace, _fused_ws_bytes(A, N, k, b_kmajor), A.device)
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_matmul_reduced_batched(_ptr(A), lda, sA, _ptr(B), ldb, sB, int(b_kmajor), ba, M, K, N,
                                            float(rho), _dtype(A), SCORE_MODES[mode], _ptr(out), ldc, sC,
                                            _out_code(out.dtype), _ptr(idx_out), ctypes.c_void_p(ws.ptr),
                                            ws.nbytes, _stream(A)))
    return out, ws


def matmul_reduced_b_norms(A: torch.Tensor, B: torch.Tensor, b_norm: torch.Tensor, rho: float,
                           out_dtype=torch.float32, out: torch.Tensor | None = None,
                           workspace: Workspace | None = None, idx_out: torch.Tensor | None = None,
                           b_kmajor: bool = False):
    """matmul_reduced in product mode with B's norms cached (see b_norms): the score reads only A."""
    ba, M, K, lda, sA = _mat(A, "A")
    bb, r, c, ldb, sB = _mat(B, "B")
    N = r if b_kmajor else c
    stride = _bn_stride(b_norm, ba, K)
    k = keep_count(rho, K)
    ws = _ensure_ws(workspace, _fused_ws_bytes(A, N, k, b_kmajor), A.device)
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_matmul_reduced_b_norms(_ptr(A), lda, sA, _ptr(B), ldb, sB, int(b_kmajor), _ptr(b_norm),
                                            stride, ba, M, K, N, float(rho), _dtype(A), _ptr(out), ldc, sC,
                                            _out_code(out.dtype), _ptr(idx_out), ctypes.c_void_p(ws.ptr),
                                            ws.nbytes, _stream(A)))
    return out, ws


def _w8(Wq: torch.Tensor, scale: torch.Tensor):
    """(batch, K, N, ldw, strideW, scale_stride) of an INT8 weight and its column scales."""
    if Wq.dtype != torch.int8:
        raise ValueError("Wq must be int8")
    bw, K, N, ldw, sW = _mat(Wq, "Wq")
    if scale.dtype != torch.float32 or not scale.is_cuda or not scale.is_contiguous():
        raise ValueError("scale must be a contiguous float32 CUDA tensor")
    if scale.dim() == 1:
        if scale.shape[0] != N:
            raise ValueError("scale must hold N values")
        return bw, K, N, ldw, sW, 0
    if tuple(scale.shape) != (bw, N):
        raise ValueError("scale must be [N] or [batch][N]")
    return bw, K, N, ldw, sW, N


def b_norms_w8(Wq: torch.Tensor, scale: torch.Tensor, out: torch.Tensor | None = None,
               status: torch.Tensor | None = None) -> torch.Tensor:
    """||W[k,:]||_2 of the dequantized INT8 weight W = Wq · diag(scale) (f32 [batch][K] or [K])."""
    bw, K, N, ldw, sW, ss = _w8(Wq, scale)
    if out is None:
        out = torch.empty((bw, K) if Wq.dim() == 3 else (K,), dtype=torch.float32, device=Wq.device)
    _check(lib().rmm_b_norms_w8(_ptr(Wq), ldw, sW, _ptr(scale), ss, bw, K, N, _ptr(out), _ptr(status), _stream(Wq)))
    return out


def pack_w8(A: torch.Tensor, Wq: torch.Tensor, scale: torch.Tensor, idx: torch.Tensor, out=None,
            status: torch.Tensor | None = None):
    """(A_S, B_S): A's kept columns and bf16(Wq[idx] · scale) — the operands rmm.gemm takes."""
    ba, M, K, lda, sA = _mat(A, "A")
    bw, K2, N, ldw, sW, ss = _w8(Wq, scale)
    if K2 != K:
        raise ValueError("A and Wq disagree on the contraction dimension")
    k = idx.shape[-1]
    kp = padded_keep(k)
    if out is None:
        A_S = torch.empty((ba, M, kp) if A.dim() == 3 else (M, kp), dtype=A.dtype, device=A.device)
        B_S = torch.empty(packed_b_shape(A.dim() == 3, ba, N, kp, False), dtype=A.dtype, device=A.device)
    else:
        A_S, B_S = out
    _check(lib().rmm_pack_w8(_ptr(A), lda, sA, _ptr(Wq), ldw, sW, _ptr(scale), ss, ba, M, K, N, _ptr(idx), k,
                             _ptr(A_S), _ptr(B_S), _ptr(status), _stream(A)))
    return A_S, B_S


def gemv_gather_w8(A: torch.Tensor, Wq: torch.Tensor, scale: torch.Tensor, idx: torch.Tensor,
                   out_dtype=torch.float32, out: torch.Tensor | None = None) -> torch.Tensor:
    """C = A[:, idx] · (Wq · diag(scale))[idx, :] straight from A (M <= 16 rows) and the INT8 weight."""
    ba, M, K, lda, sA = _mat(A, "A")
    bw, K2, N, ldw, sW, ss = _w8(Wq, scale)
    if K2 != K:
        raise ValueError("A and Wq disagree on the contraction dimension")
    k = idx.shape[-1]
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_gemv_gather_w8(_ptr(A), lda, sA, _ptr(Wq), ldw, sW, _ptr(scale), ss, ba, M, K, N, _ptr(idx), k,
                                    _ptr(out), ldc, sC, _out_code(out.dtype), _stream(A)))
    return out


def matmul_reduced_w8(A: torch.Tensor, Wq: torch.Tensor, scale: torch.Tensor, rho: float,
                      b_norm: torch.Tensor | None = None, mode: str = "product", out_dtype=torch.float32,
                      out: torch.Tensor | None = None, workspace: Workspace | None = None,
                      idx_out: torch.Tensor | None = None):
    """matmul_reduced on an INT8 weight W = Wq · diag(scale); product mode needs b_norm (b_norms_w8)."""
    ba, M, K, lda, sA = _mat(A, "A")
    bw, K2, N, ldw, sW, ss = _w8(Wq, scale)
    if K2 != K:
        raise ValueError("A and Wq disagree on the contraction dimension")
    bn_stride = 0
    if b_norm is not None:
        bn_stride = _bn_stride(b_norm, ba, K)
    elif SCORE_MODES[mode] == 0:
        raise ValueError("product mode needs b_norm (b_norms_w8)")
    k = keep_count(rho, K)
    ws = _ensure_ws(workspace, workspace_size_for(ba, M, K, N, k, A.dtype), A.device)
    if out is None:
        out = torch.empty((ba, M, N) if A.dim() == 3 else (M, N), dtype=out_dtype, device=A.device)
    _, _, _, ldc, sC = _mat(out, "C")
    _check(lib().rmm_matmul_reduced_w8(_ptr(A), lda, sA, _ptr(Wq), ldw, sW, _ptr(scale), ss, _ptr(b_norm), bn_stride,
                                       ba, M, K, N, float(rho), _dtype(A), SCORE_MODES[mode], _ptr(out), ldc, sC,
                                       _out_code(out.dtype), _ptr(idx_out), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                       _stream(A)))
    return out, ws


def qk_reduced(Q: torch.Tensor, Kmat: torch.Tensor, rho: float, mode: str = "product", out_dtype=torch.float32,
               out: torch.Tensor | None = None, workspace: Workspace | None = None,
               idx_out: torch.Tensor | None = None):
    """S = Q·Kᵀ per head, reduced over head_dim. Q [bh][S_q][d], Kmat [bh][S_k][d]."""
    bh, S_q, d = Q.shape
    S_k = Kmat.shape[1]
    k = keep_count(rho, d)
    ws = _ensure_ws(workspace, _fused_ws_bytes(Q, S_k, k, True), Q.device)
    if out is None:
        out = torch.empty(bh, S_q, S_k, dtype=out_dtype, device=Q.device)
    _check(lib().rmm_qk_reduced(_ptr(Q), _ptr(Kmat), bh, S_q, S_k, d, float(rho), _dtype(Q), SCORE_MODES[mode],
                                _ptr(out), _out_code(out.dtype), _ptr(idx_out), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                _stream(Q)))
    return out, ws


def pv_reduced(P: torch.Tensor, V: torch.Tensor, rho: float, mode: str = "product", out_dtype=torch.float32,
               out: torch.Tensor | None = None, workspace: Workspace | None = None,
               idx_out: torch.Tensor | None = None):
    """O = P·V per head, reduced over the keys. P [bh][S_q][S_k], V [bh][S_k][d]."""
    bh, S_q, S_k = P.shape
    d = V.shape[2]
    k = keep_count(rho, S_k)
    ws = _ensure_ws(workspace, _fused_ws_bytes(P, d, k, False), P.device)
    if out is None:
        out = torch.empty(bh, S_q, d, dtype=out_dtype, device=P.device)
    _check(lib().rmm_pv_reduced(_ptr(P), _ptr(V), bh, S_q, S_k, d, float(rho), _dtype(P), SCORE_MODES[mode],
                                _ptr(out), _out_code(out.dtype), _ptr(idx_out), ctypes.c_void_p(ws.ptr), ws.nbytes,
                                _stream(P)))
    return out, ws


# ---------------------------------------------------------------- P·V with its softmax producer
def softmax_row_stats(L: torch.Tensor, scale: float = 1.0, causal: bool = True, out: torch.Tensor | None = None,
                      status: torch.Tensor | None = None) -> torch.Tensor:
    """[bh][S_q][2] f32: max of scale·log2(e)·L over each row's visible keys, and 1 / sum exp2(. - max)."""
    bh, S_q, S_k = L.shape
    if not L.is_contiguous():
        raise ValueError("L must be contiguous")
    if out is None:
        out = torch.empty(bh, S_q, 2, dtype=torch.float32, device=L.device)
    _check(lib().rmm_softmax_row_stats(_ptr(L), _dtype(L), float(scale), int(causal), bh, S_q, S_k, _ptr(out),
                                       _ptr(status), _stream(L)))
    return out


def softmax_score(L: torch.Tensor, stats: torch.Tensor, V: torch.Tensor | None = None, scale: float = 1.0,
                  causal: bool = True, score: bool = True, P: torch.Tensor | None = None,
                  s: torch.Tensor | None = None, status: torch.Tensor | None = None):
    """(P, s): P = softmax(scale·L) stored bf16, and (score=True) s[b][k] =
    ||P[b][:, k]|| · ||V[b][k, :]|| (or ||P[b][:, k]|| without V)."""
    bh, S_q, S_k = L.shape
    if not L.is_contiguous():
        raise ValueError("L must be contiguous")
    if V is not None and (V.dtype != torch.bfloat16 or not V.is_contiguous() or V.shape[:2] != (bh, S_k)):
        raise ValueError("V must be a contiguous bf16 [bh][S_k][d] tensor")
    d = V.shape[2] if V is not None else 0
    if P is None:
        P = torch.empty(bh, S_q, S_k, dtype=torch.bfloat16, device=L.device)
    if score and s is None:
        s = torch.empty(bh, S_k, dtype=torch.float32, device=L.device)
    _check(lib().rmm_softmax_score(_ptr(L), _dtype(L), float(scale), int(causal), _ptr(stats), _ptr(V), d, bh, S_q,
                                   S_k, _ptr(P), _ptr(s if score else None), _ptr(status), _stream(L)))
    return P, (s if score else None)


def pv_softmax_workspace_size(bh: int, S_q: int, S_k: int, d: int, k_keep: int) -> int:
    return int(lib().rmm_pv_softmax_workspace_size(bh, S_q, S_k, d, k_keep))


def pv_softmax_reduced(L: torch.Tensor, V: torch.Tensor, rho: float, scale: float = 1.0, causal: bool = True,
                       mode: str = "product", out_dtype=torch.float32, P: torch.Tensor | None = None,
                       out: torch.Tensor | None = None, workspace: Workspace | None = None,
                       idx_out: torch.Tensor | None = None):
    """O ≈ P·V with P = softmax(scale·L) written by the call (bf16) and scored
    as it is written. Returns (O, P, workspace)."""
    bh, S_q, S_k = L.shape
    d = V.shape[2]
    if not L.is_contiguous() or not V.is_contiguous() or V.dtype != torch.bfloat16:
        raise ValueError("L must be contiguous and V a contiguous bf16 tensor")
    k = keep_count(rho, S_k)
    ws = _ensure_ws(workspace, pv_softmax_workspace_size(bh, S_q, S_k, d, k), L.device)
    if P is None:
        P = torch.empty(bh, S_q, S_k, dtype=torch.bfloat16, device=L.device)
    if out is None:
        out = torch.empty(bh, S_q, d, dtype=out_dtype, device=L.device)
    _check(lib().rmm_pv_softmax_reduced(_ptr(L), _dtype(L), float(scale), int(causal), _ptr(V), bh, S_q, S_k, d,
                                        float(rho), SCORE_MODES[mode], _ptr(P), _ptr(out), _out_code(out.dtype),
                                        _ptr(idx_out), ctypes.c_void_p(ws.ptr), ws.nbytes, _stream(L)))
    return out, P, ws


def set_wait_limit_ns(ns: int):
    lib().rmm_set_wait_limit_ns(int(ns))


def set_stall_producer_for_test(on: bool):
    lib().rmm_set_stall_producer_for_test(int(bool(on)))


def set_gemm_cta_group(cta_group: int) -> int:
    """2 = 2-SM MMAs on CTA pairs (default), 1 = one SM per tile; returns the previous value."""
    return int(lib().rmm_set_gemm_cta_group(int(cta_group)))


def launch_count() -> int:
    return int(lib().rmm_launch_count())


def set_debug(on: bool) -> bool:
    """Debug checks (kept indices validated on the device before a stage call
    reads through them; fused calls report their device status directly).
    Returns the previous setting."""
    return bool(lib().rmm_set_debug(int(bool(on))))


def set_gemm_events(start: torch.cuda.Event | None, stop: torch.cuda.Event | None):
    """Record `start`/`stop` immediately around every GEMM kernel launch (None, None clears)."""
    def handle(e):
        if e is None:
            return ctypes.c_void_p(0)
        if not e.cuda_event:  # torch creates the CUDA event on its first record
            e.record()
        return ctypes.c_void_p(e.cuda_event)

    lib().rmm_set_gemm_events(handle(start), handle(stop))


def matmul_reduced_noalloc(A: torch.Tensor, B: torch.Tensor, rho: float, mode: str = "product",
                           out_dtype=torch.float32, out: torch.Tensor | None = None,
                           idx_out: torch.Tensor | None = None, status: torch.Tensor | None = None):
    """C ≈ A·B like matmul_reduced, but with the library's static 32 MiB device
    scratch instead of a workspace, for callers that must not allocate device
    memory (only C is allocated here, and only when `out` is None)."""
    _, M, K, lda, _ = _mat(A, "A")
    _, r, N, ldb, _ = _mat(B, "B")
    if out is None:
        out = torch.empty(M, N, dtype=out_dtype, device=A.device)
    _, _, _, ldc, _ = _mat(out, "C")
    _check(lib().rmm_matmul_reduced_noalloc(_ptr(A), lda, _ptr(B), ldb, M, K, N, float(rho), _dtype(A),
                                            SCORE_MODES[mode], _ptr(out), ldc, _out_code(out.dtype), _ptr(idx_out),
                                            _ptr(status), _stream(A)))
    return out
