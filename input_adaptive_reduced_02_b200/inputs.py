"""Seeded synthetic inputs shaped like the workloads the RMM pages evaluate on.

This module only draws random matrices. It holds none of the method's arithmetic
(no norms, no scores, no selection, no products), so both the CUDA path and the
fp64 oracle can take their inputs from it.

Every generator uses torch's Philox generator on the requested device, seeded
explicitly, then rounds to the storage dtype (bf16 with round-to-nearest-even).
The same tensor is handed to the library and, copied to the host, to the oracle.

Workload shapes follow the application sites named on the gist.science summary
page "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
LLM Inference" (Resumo Técnico, Metodologia, "Escopo de Aplicação"): Q·Kᵀ reduced
over the head dimension, P·V reduced over the token (key) dimension, and X·W
reduced over the hidden dimension. The value distributions (outlier channels,
causal softmax, SiLU activations) are the plainest synthetic stand-ins for the
activations of the 1B-70B LLaMA/Qwen models the pages evaluate (Resultados).
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def lognormal_slices_f32(M: int = 64, K: int = 256, N: int = 64, seed: int = 0,
                         device="cpu"):
    """fp32 A (M×K), B (K×N): i.i.d. N(0,1) entries; column k of A and row k of B
    each multiplied by an independent exp(N(0,1)) factor so that slice importance
    varies from slice to slice."""
    g = _gen(seed, device)
    A = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    B = torch.randn(K, N, generator=g, device=device, dtype=torch.float32)
    a_scale = torch.exp(torch.randn(K, generator=g, device=device, dtype=torch.float32))
    b_scale = torch.exp(torch.randn(K, generator=g, device=device, dtype=torch.float32))
    return (A * a_scale[None, :]).contiguous(), (B * b_scale[:, None]).contiguous()


def outlier_activations(M: int, K: int, outlier_frac: float, factor: float,
                        seed: int, device="cpu", dtype=torch.bfloat16):
    """X (M×K): N(0,1) with round(outlier_frac·K) seeded hidden channels (columns)
    multiplied by `factor`. Returns (X, outlier_channel_indices)."""
    g = _gen(seed, device)
    X = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    n_out = int(round(outlier_frac * K))
    ch = torch.randperm(K, generator=g, device=device)[:n_out]
    if n_out:
        X[:, ch] *= factor
    return X.to(dtype).contiguous(), ch


def int8_weight(K: int, N: int, std: float = 0.02, seed: int = 0, device="cpu"):
    """A weight given as INT8 codes and one f32 scale per output column:
    Wq [K][N] int8 = round(N(0, 40²)) clipped to [-127, 127]; scale [N] =
    std/40 · (1 + 0.1·N(0,1)), so Wq · scale has entries of about N(0, std²)."""
    g = _gen(seed, device)
    q = torch.randn(K, N, generator=g, device=device, dtype=torch.float32) * 40.0
    Wq = q.round().clamp(-127, 127).to(torch.int8).contiguous()
    scale = (std / 40.0) * (1.0 + 0.1 * torch.randn(N, generator=g, device=device, dtype=torch.float32))
    return Wq, scale.contiguous()


def gaussian(shape, std: float, seed: int, device="cpu", dtype=torch.bfloat16):
    """N(0, std²) entries of the given shape."""
    g = _gen(seed, device)
    W = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        W *= std
    return W.to(dtype).contiguous()


def linear_projection(M: int = 4096, K: int = 4096, N: int = 4096, seed: int = 0,
                      device="cpu"):
    """X (M×K) bf16 N(0,1) with 1% outlier hidden channels ×20; W (K×N) bf16 N(0, 0.02²)."""
    X, _ = outlier_activations(M, K, 0.01, 20.0, seed, device)
    W = gaussian((K, N), 0.02, seed + 1, device)
    return X, W


def attention_qk(bh: int = 32, S: int = 4096, d: int = 128, n_outlier: int = 4,
                 factor: float = 8.0, seed: int = 0, device="cpu"):
    """Q, K [bh][S][d] bf16 N(0,1); the same `n_outlier` seeded head_dim channels
    are multiplied by `factor` in both Q and K."""
    g = _gen(seed, device)
    Q = torch.randn(bh, S, d, generator=g, device=device, dtype=torch.float32)
    Km = torch.randn(bh, S, d, generator=g, device=device, dtype=torch.float32)
    ch = torch.randperm(d, generator=g, device=device)[:n_outlier]
    Q[:, :, ch] *= factor
    Km[:, :, ch] *= factor
    return Q.to(torch.bfloat16).contiguous(), Km.to(torch.bfloat16).contiguous()


def causal_softmax_probs(S_q: int, S_k: int, temperature: float, g: torch.Generator,
                         device, out: torch.Tensor, row_chunk: int = 2048):
    """Fill `out` ([S_q][S_k] bf16) with a row softmax, computed in fp32, of
    temperature·N(0,1) logits under a causal mask (key k visible to query q iff
    k ≤ q + S_k − S_q). Rows are drawn in chunks to bound temporary memory."""
    offset = S_k - S_q
    cols = torch.arange(S_k, device=device)
    for r0 in range(0, S_q, row_chunk):
        r1 = min(S_q, r0 + row_chunk)
        logits = torch.randn(r1 - r0, S_k, generator=g, device=device, dtype=torch.float32)
        logits *= temperature
        rows = torch.arange(r0, r1, device=device)
        masked = cols[None, :] > (rows[:, None] + offset)
        logits.masked_fill_(masked, float("-inf"))
        out[r0:r1].copy_(torch.softmax(logits, dim=1).to(torch.bfloat16))
        del logits, masked
    return out


def attention_pv(bh: int = 32, S: int = 8192, d: int = 128, temperature: float = 3.0,
                 seed: int = 0, device="cpu", heads=None):
    """P [bh][S][S] bf16 (causal row softmax of temperature·N(0,1) logits, fp32
    softmax then bf16), V [bh][S][d] bf16 N(0,1). Head h draws from seed + h, so a
    subset of heads (`heads`) can be regenerated exactly on its own."""
    heads = list(range(bh)) if heads is None else list(heads)
    P = torch.empty(len(heads), S, S, device=device, dtype=torch.bfloat16)
    V = torch.empty(len(heads), S, d, device=device, dtype=torch.bfloat16)
    for j, h in enumerate(heads):
        g = _gen(seed * 1000003 + h, device)
        causal_softmax_probs(S, S, temperature, g, device, P[j])
        V[j].copy_(torch.randn(S, d, generator=g, device=device, dtype=torch.float32)
                   .to(torch.bfloat16))
    return P, V


def attention_logits(bh: int = 32, S: int = 8192, d: int = 128, temperature: float = 3.0, seed: int = 0,
                     device="cpu", dtype=torch.bfloat16, S_q: int | None = None):
    """Logits L [bh][S_q][S] = temperature·N(0,1) (stored in `dtype`) and V
    [bh][S][d] bf16 N(0,1): the inputs of P·V when P is produced from its
    logits (P = causal row softmax of L). Head h draws from seed + h."""
    S_q = S if S_q is None else S_q
    L = torch.empty(bh, S_q, S, device=device, dtype=dtype)
    V = torch.empty(bh, S, d, device=device, dtype=torch.bfloat16)
    for h in range(bh):
        g = _gen(seed * 1000003 + h, device)
        for r0 in range(0, S_q, 1024):
            r1 = min(S_q, r0 + 1024)
            L[h, r0:r1].copy_(temperature * torch.randn(r1 - r0, S, generator=g, device=device, dtype=torch.float32))
        V[h].copy_(torch.randn(S, d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16))
    return L, V


def mlp_up(M: int = 2048, K: int = 8192, N: int = 28672, seed: int = 0, device="cpu"):
    """Up-projection: X (M×K) bf16 N(0,1) with 0.5% outlier channels ×20; W (K×N) N(0, 0.01²)."""
    X, _ = outlier_activations(M, K, 0.005, 20.0, seed, device)
    W = gaussian((K, N), 0.01, seed + 1, device)
    return X, W


def mlp_down(M: int = 2048, K: int = 28672, N: int = 8192, seed: int = 0, device="cpu"):
    """Down-projection: H = SiLU(N(0,1)) (M×K) bf16; W (K×N) bf16 N(0, 0.01²)."""
    g = _gen(seed, device)
    H = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    H = torch.nn.functional.silu(H).to(torch.bfloat16).contiguous()
    W = gaussian((K, N), 0.01, seed + 1, device)
    return H, W


#: The workloads the library is measured and parity-checked on.
WORKLOADS = {
    "f32_64x256x64": dict(kind="single", M=64, K=256, N=64, dtype="f32", rhos=(0.5,)),
    "linear_4096": dict(kind="single", M=4096, K=4096, N=4096, dtype="bf16",
                        rhos=(0.3, 0.5, 0.7, 0.9, 1.0)),
    "qk_32x4096x128": dict(kind="qk", bh=32, S=4096, d=128, dtype="bf16", rhos=(0.5,)),
    "pv_32xSx128": dict(kind="pv", bh=32, S=(8192, 16384, 32768), d=128, dtype="bf16",
                        rhos=(0.3, 0.5, 0.7)),
    "mlp_up_2048x8192x28672": dict(kind="single", M=2048, K=8192, N=28672, dtype="bf16",
                                   rhos=(0.5, 0.7, 0.9)),
    "mlp_down_2048x28672x8192": dict(kind="single", M=2048, K=28672, N=8192, dtype="bf16",
                                     rhos=(0.5, 0.7, 0.9)),
}
