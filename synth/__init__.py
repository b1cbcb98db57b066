"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and rounds them to bf16; it holds none
of the quantization, GEMM or EAR/KL arithmetic, so both the CUDA library and
the CPU oracle can be fed from it without sharing any of the method.

Recipes (they stand in for the pages' Qwen3 / Llama-3.3 weights, activations
and calibration logits, which are not available here):

* weights: per row and per 128-wide group along K, sigma_g = exp(U(ln 0.005,
  ln 0.05)), mu_g ~ N(0, (0.5 sigma_g)^2), w ~ N(mu_g, sigma_g^2); then each
  element independently, with probability 0.001, is multiplied by 8
  (outliers).  The second argument of N(.,.) in the recipe is the std.
* activations X ~ N(0, 1).
* logits: reference a ~ N(0, 3^2); per row one token u ~ U{0..V-1} gets
  a[u] = max(a) + 6 + G with G ~ Gumbel(0, 1) (a confident next token);
  quantized-model logits b = a + N(0, 0.05^2).
* All values are drawn in binary64 (CPU, numpy PCG64) or binary32 (device,
  torch Philox) and rounded to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import numpy as np

GROUP = 128

# Seeds used by the tests and the benchmark.
SEED_WEIGHTS = 1000
SEED_X = 2000
SEED_LOGITS = 3000
SEED_LOGIT_NOISE = 3001


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to bf16 (nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    return ((u + bias) >> 16).astype(np.uint16)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """binary64 -> binary32 (nearest even) -> bf16 (nearest even)."""
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float64).astype(np.float32))


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# CPU generators (numpy PCG64, binary64)
# ----------------------------------------------------------------------------

def weights(N: int, K: int, seed: int = SEED_WEIGHTS, outlier_p: float = 0.001) -> np.ndarray:
    """Skewed-Gaussian grouped weights, [N, K] bf16 bits."""
    assert K % GROUP == 0
    G = K // GROUP
    rng = np.random.default_rng(seed)
    sigma = np.exp(rng.uniform(np.log(0.005), np.log(0.05), size=(N, G)))
    mu = rng.normal(0.0, 0.5 * sigma)
    w = mu[:, :, None] + sigma[:, :, None] * rng.standard_normal((N, G, GROUP))
    w = w.reshape(N, K)
    if outlier_p > 0:
        w = np.where(rng.random((N, K)) < outlier_p, 8.0 * w, w)
    return to_bf16_bits(w)


def activations(M: int, K: int, seed: int = SEED_X) -> np.ndarray:
    """X ~ N(0, 1), [M, K] bf16 bits."""
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal((M, K)))


def calibration(T: int, K: int, seed: int = SEED_X, rho: float = 0.9) -> np.ndarray:
    """Calibration rows [T, K] bf16 bits whose neighbouring inputs are
    correlated: x_k = rho x_{k-1} + sqrt(1 - rho^2) z_k, z ~ N(0, 1) (standing
    in for the pages' FineWeb-Edu calibration tokens)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, K))
    x = np.empty_like(z)
    x[:, 0] = z[:, 0]
    for k in range(1, K):
        x[:, k] = rho * x[:, k - 1] + np.sqrt(1 - rho**2) * z[:, k]
    return to_bf16_bits(x)


def logits(T: int, V: int, seed: int = SEED_LOGITS, noise_seed: int = SEED_LOGIT_NOISE,
           std: float = 3.0, peak: float = 6.0, noise_std: float = 0.05):
    """(reference, quantized) logit rows, each [T, V] bf16 bits."""
    rng = np.random.default_rng(seed)
    a = std * rng.standard_normal((T, V))
    top = rng.integers(0, V, size=T)
    gum = rng.gumbel(0.0, 1.0, size=T)
    a[np.arange(T), top] = a.max(axis=1) + peak + gum
    a_bits = to_bf16_bits(a)
    a_val = bf16_bits_to_f32(a_bits).astype(np.float64)
    nrng = np.random.default_rng(noise_seed)
    b_bits = to_bf16_bits(a_val + noise_std * nrng.standard_normal((T, V)))
    return a_bits, b_bits


# ----------------------------------------------------------------------------
# Device generators (torch Philox on the GPU; same recipes, binary32 draws).
# Used where the CPU generators would take too long (full-size benchmark
# inputs).  They give different numbers from the CPU ones for the same seed.
# ----------------------------------------------------------------------------

def _gen(device, seed):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weights_torch(N: int, K: int, seed: int = SEED_WEIGHTS, device="cuda", outlier_p: float = 0.001):
    import torch
    assert K % GROUP == 0
    G = K // GROUP
    g = _gen(device, seed)
    out = torch.empty((N, K), dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 24) // K)
    for r0 in range(0, N, rows):
        r1 = min(N, r0 + rows)
        n = r1 - r0
        u = torch.rand((n, G), generator=g, device=device, dtype=torch.float32)
        sigma = torch.exp(np.log(0.005) + u * (np.log(0.05) - np.log(0.005)))
        mu = 0.5 * sigma * torch.randn((n, G), generator=g, device=device)
        w = mu[:, :, None] + sigma[:, :, None] * torch.randn((n, G, GROUP), generator=g, device=device)
        w = w.reshape(n, K)
        if outlier_p > 0:
            mask = torch.rand((n, K), generator=g, device=device) < outlier_p
            w = torch.where(mask, 8.0 * w, w)
        out[r0:r1] = w.to(torch.bfloat16)
    return out


def activations_torch(M: int, K: int, seed: int = SEED_X, device="cuda"):
    import torch
    g = _gen(device, seed)
    return torch.randn((M, K), generator=g, device=device).to(torch.bfloat16)


def logits_torch(T: int, V: int, seed: int = SEED_LOGITS, noise_seed: int = SEED_LOGIT_NOISE,
                 device="cuda", std: float = 3.0, peak: float = 6.0, noise_std: float = 0.05):
    import torch
    g = _gen(device, seed)
    gn = _gen(device, noise_seed)
    a = torch.empty((T, V), dtype=torch.bfloat16, device=device)
    b = torch.empty((T, V), dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 26) // V)
    for r0 in range(0, T, rows):
        r1 = min(T, r0 + rows)
        n = r1 - r0
        x = std * torch.randn((n, V), generator=g, device=device)
        top = torch.randint(0, V, (n,), generator=g, device=device)
        u = torch.rand((n,), generator=g, device=device).clamp_min(1e-30)
        gum = -torch.log(-torch.log(u))
        x[torch.arange(n, device=device), top] = x.max(dim=1).values + peak + gum
        xa = x.to(torch.bfloat16)
        a[r0:r1] = xa
        b[r0:r1] = (xa.float() + noise_std * torch.randn((n, V), generator=gn, device=device)).to(torch.bfloat16)
    return a, b
