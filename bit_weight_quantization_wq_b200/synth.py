"""Seeded synthetic inputs for the quantized linear layer.

This module feeds both the CUDA path and the CPU oracle. It holds none of the method's
arithmetic (no abs-max, step, rounding to codes, packing or GEMM): only random draws,
the bf16 rounding of those draws, and the construction of the low-rank factors that a
SVDQuant-style model ships next to its residual weights.

Workloads (standing in for the pages' Wan-Dancer-14B / FLUX weights, which are not here):
  * weights  ~ N(0, sigma^2), with round(0.001 * N * K) outliers at distinct positions,
    each +-1 (p = 1/2) times U(0.2, 0.5);
  * activations x ~ N(0, 1), optionally with a few outlier channels scaled by 20;
  * bias ~ N(0, 0.01^2).
Every tensor is rounded to bf16 (round to nearest even) and returned as its uint16 bit
patterns (numpy has no bf16).
"""
from __future__ import annotations

import numpy as np

# per-tensor bit-width distribution of the mixed-precision DiT block stack: the 525-tensor
# histogram {3: 1, 4: 111, 5: 288, 6: 121, 7: 4} at 5.0 BPW, as fractions
MIXED_BITS = (3, 4, 5, 6, 7)
MIXED_PROBS = (0.002, 0.211, 0.549, 0.230, 0.008)

# one DiT block of the 5120-hidden stack: 8 attention projections, FFN up and down
BLOCK_SHAPES = [(5120, 5120)] * 8 + [(13824, 5120), (5120, 13824)]


def rng_for(config: int, block: int = 0, idx: int = 0) -> np.random.Generator:
    """Independent PCG64 stream per (config, block, tensor index); config seed is 1000 + c."""
    return np.random.default_rng([1000 + config, block, idx])


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def weight(rng: np.random.Generator, N: int, K: int, sigma: float,
           outlier_frac: float = 1e-3, outlier_cols: int = 0) -> np.ndarray:
    """N x K bf16 weight: Gaussian body plus sparse +-U(0.2, 0.5) outliers.

    outlier_cols > 0 concentrates the outliers in that many random input columns
    (positions drawn without replacement inside those columns, capped at all of them).
    """
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(sigma)
    n_out = int(round(outlier_frac * N * K))
    if outlier_cols > 0:
        cols = rng.choice(K, size=outlier_cols, replace=False)
        n_out = min(n_out, N * outlier_cols)
        flat = rng.choice(N * outlier_cols, size=n_out, replace=False)
        rows, ci = flat // outlier_cols, flat % outlier_cols
        pos = rows * K + cols[ci]
    else:
        pos = rng.choice(N * K, size=n_out, replace=False)
    sign = np.where(rng.random(n_out) < 0.5, -1.0, 1.0)
    mag = rng.uniform(0.2, 0.5, n_out)
    w.reshape(-1)[pos] = (sign * mag).astype(np.float32)
    return f32_to_bf16_bits(w)


def activations(rng: np.random.Generator, M: int, K: int, outlier_channels: int = 0,
                outlier_scale: float = 20.0) -> np.ndarray:
    """M x K bf16 activations ~ N(0, 1); `outlier_channels` random columns scaled up."""
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outlier_channels:
        ch = rng.choice(K, size=outlier_channels, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def bias(rng: np.random.Generator, N: int, sigma: float = 0.01) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(sigma))


def torch_generator(config: int, block: int = 0, idx: int = 0, device="cuda"):
    """A torch generator on `device` seeded from (config, block, tensor index), for the
    workloads too large to draw on the host (the 40-block stack and the 49-block model)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(((1000 + config) * 1_000_003 + block) * 1009 + idx)
    return g


def weight_torch(gen, N: int, K: int, sigma: float, outlier_frac: float = 1e-3, device="cuda"):
    """The :func:`weight` recipe drawn with a torch generator on the device: N x K bf16 torch
    tensor, N(0, sigma^2) body with round(outlier_frac * N * K) distinct outlier positions,
    each +-1 (p = 1/2) times U(0.2, 0.5); fp32 draws rounded to bf16 (nearest even)."""
    import torch
    w = torch.randn(N, K, device=device, generator=gen, dtype=torch.float32) * sigma
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        pos = torch.randperm(N * K, device=device, generator=gen)[:n_out]
        sign = torch.where(torch.rand(n_out, device=device, generator=gen) < 0.5, -1.0, 1.0)
        mag = torch.rand(n_out, device=device, generator=gen, dtype=torch.float64) * 0.3 + 0.2
        w.view(-1)[pos] = (sign * mag).to(torch.float32)
    return w.to(torch.bfloat16)


def lowrank_split(W_bits: np.ndarray, rank: int, rng: np.random.Generator, power_iters: int = 4):
    """Split W into a rank-r bf16 branch and a bf16 residual, as an SVDQuant model ships it.

    W ~= U_r S_r V_r^T from a randomized subspace iteration (fp64). L1 = bf16(V_r S_r)
    (K x r), L2 = bf16(U_r^T) (r x N), and the residual R = bf16(W - (L1 L2)^T) computed in
    fp64 from the rounded factors. The residual is what gets quantized; L1 and L2 are the
    16-bit branch. The split of S between the factors only affects rounding.
    Returns (L1_bits, L2_bits, R_bits).
    """
    W = bf16_bits_to_f32(W_bits).astype(np.float64)
    N, K = W.shape
    p = min(rank + 16, min(N, K))
    Q = rng.standard_normal((K, p))
    Y = W @ Q
    for _ in range(power_iters):
        Y, _ = np.linalg.qr(Y)
        Z, _ = np.linalg.qr(W.T @ Y)
        Y = W @ Z
    Qy, _ = np.linalg.qr(Y)
    B = Qy.T @ W                                   # p x K
    Ub, s, Vt = np.linalg.svd(B, full_matrices=False)
    U = Qy @ Ub[:, :rank]                          # N x r
    L1 = (Vt[:rank].T * s[:rank]).astype(np.float32)   # K x r
    L2 = U.T.astype(np.float32)                         # r x N
    L1_bits, L2_bits = f32_to_bf16_bits(L1), f32_to_bf16_bits(L2)
    approx = bf16_bits_to_f32(L1_bits).astype(np.float64) @ bf16_bits_to_f32(L2_bits).astype(np.float64)
    R = W - approx.T
    return L1_bits, L2_bits, f32_to_bf16_bits(R.astype(np.float32))


# ----------------------------------------------------------------------------- workloads

def single_linear(config: int = 1, N: int = 256, K: int = 512, M: int = 64, sigma: float = 0.02,
                  with_bias: bool = True):
    """Single 4-bit linear: W N x K, x M x K, bias N (the 256x512, M=64 case by default)."""
    W = weight(rng_for(config, 0, 0), N, K, sigma)
    x = activations(rng_for(config, 0, 1), M, K)
    b = bias(rng_for(config, 0, 2), N) if with_bias else None
    return W, x, b


FLUX_SHAPES = [(3072, 3072), (12288, 3072), (3072, 12288)]


def flux_linears(M: int = 4096, rank: int = 32, config: int = 2, shapes=None):
    """FLUX-like DiT linears with a rank-32 bf16 branch and a quantized residual.

    For each (N, K): W ~ N(0, 0.02^2) with 0.1% outliers concentrated in 8 input columns;
    x M x K ~ N(0, 1) with 4 outlier channels x20; bias ~ N(0, 0.01^2); L1/L2/R from
    :func:`lowrank_split`. Returns a list of dicts with keys W, R, L1, L2, x, bias, N, K, M.
    """
    out = []
    for i, (N, K) in enumerate(shapes or FLUX_SHAPES):
        W = weight(rng_for(config, i, 0), N, K, 0.02, outlier_cols=8)
        L1, L2, R = lowrank_split(W, rank, rng_for(config, i, 3)) if rank > 0 else (None, None, W)
        x = activations(rng_for(config, i, 1), M, K, outlier_channels=4)
        b = bias(rng_for(config, i, 2), N)
        out.append(dict(W=W, R=R, L1=L1, L2=L2, x=x, bias=b, N=N, K=K, M=M))
    return out


WAN_SHAPES = [(5120, 5120), (13824, 5120)]


def wan_weight(i: int, config: int = 3):
    N, K = WAN_SHAPES[i]
    return weight(rng_for(config, i, 0), N, K, 0.015)


def wan_x(M: int, K: int = 5120, config: int = 3, tag: int = 0):
    return activations(rng_for(config, 100 + tag, M), M, K)


def mixed_bits(n_tensors: int, config: int = 4, block: int = 0) -> list:
    """Per-tensor bit widths drawn i.i.d. from the mixed-precision histogram."""
    rng = rng_for(config, block, 999)
    return [int(b) for b in rng.choice(MIXED_BITS, size=n_tensors, p=MIXED_PROBS)]
