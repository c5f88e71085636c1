"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds random-number recipes only -- none of the compression or
product arithmetic.  The inputs of tests and the smoke check are drawn on the
host with a CPU ``torch.Generator`` so that the CPU oracle and the GPU
library see identical BF16 bit patterns; arrays come back as numpy
``uint16`` bit patterns (row-major) so that neither side depends on the
other's tensor types.  The benchmark's 32-layer stack is drawn on the device
(same distributions, a CUDA generator; see the end of the file).

The shapes stand in for the Llama-3.1-8B MLP projections that the Unweight
pages measure on (gate/up ``[14336, 4096]``, down ``[4096, 14336]``); those
trained weights are not available, so values are N(0, sigma) with a few
heavy-tailed outliers, which reproduces the exponent statistics the pages
describe (a handful of exponents dominate; ~2.6 bits of information).
"""
from __future__ import annotations

import numpy as np
import torch

X_SEED_OFFSET = 1_000_000


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def to_bits(t: torch.Tensor) -> np.ndarray:
    """float32 tensor -> BF16 (round to nearest even) bit patterns, uint16."""
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_float(b: np.ndarray) -> np.ndarray:
    """BF16 bit patterns -> float32 values (exact widening)."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def gaussian_weight(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """W[N, K] ~ N(0, std), rounded to BF16."""
    g = _gen(seed)
    return to_bits(torch.randn(N, K, generator=g, dtype=torch.float32) * std)


def student_t3(n: int, g: torch.Generator) -> torch.Tensor:
    """Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)."""
    z = torch.randn(n, generator=g, dtype=torch.float64)
    c = torch.randn(3, n, generator=g, dtype=torch.float64).pow(2).sum(0)
    return (z / torch.sqrt(c / 3.0)).to(torch.float32)


def weight_with_tail(N: int, K: int, seed: int, std: float = 0.02, frac: float = 0.001) -> np.ndarray:
    """N(0, std) weights where a fraction `frac` of the elements (seeded
    positions) is replaced by std * t_3 (heavy tail)."""
    g = _gen(seed)
    w = torch.randn(N * K, generator=g, dtype=torch.float32) * std
    cnt = int(round(frac * N * K))
    if cnt:
        pos = torch.randperm(N * K, generator=g)[:cnt]
        w[pos] = std * student_t3(cnt, g)
    return to_bits(w.view(N, K))


def weight_with_verbatim_rows(N: int, K: int, seed: int, std: float = 0.02,
                              frac_groups: float = 0.005, scale_pow2: int = 12) -> np.ndarray:
    """N(0, std) weights; in round(frac_groups * G) distinct 64-weight groups
    (seeded choice) one uniformly chosen element is multiplied by
    2**scale_pow2 (exact in BF16), which pushes its exponent far outside the
    common range."""
    g = _gen(seed)
    w = torch.randn(N * K, generator=g, dtype=torch.float32) * std
    w = w.to(torch.bfloat16).to(torch.float32)
    G = N * K // 64
    cnt = int(round(frac_groups * G))
    if cnt:
        groups = torch.randperm(G, generator=g)[:cnt]
        within = torch.randint(0, 64, (cnt,), generator=g)
        pos = groups * 64 + within
        w[pos] = w[pos] * float(2 ** scale_pow2)
    return to_bits(w.view(N, K))


def activations(M: int, K: int, seed: int) -> np.ndarray:
    """X[M, K] ~ N(0, 1), rounded to BF16."""
    g = _gen(seed)
    return to_bits(torch.randn(M, K, generator=g, dtype=torch.float32))


def all_bf16_patterns() -> np.ndarray:
    """Every 16-bit pattern once, as a [1024, 64] matrix (row-major)."""
    return np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(1024, 64)


def layer_stds(n_layers: int = 32, seed: int = 999) -> np.ndarray:
    """Per-layer weight std ~ U(0.015, 0.03)."""
    g = _gen(seed)
    return (torch.rand(n_layers, generator=g, dtype=torch.float64) * 0.015 + 0.015).numpy()


# --------------------------------------------------------------------------
# The named workloads.
# --------------------------------------------------------------------------
def small_matrix():
    """W[512, 2048], seed 0, 0.5% of groups forced verbatim; X[4, 2048]."""
    W = weight_with_verbatim_rows(512, 2048, seed=0)
    X = activations(4, 2048, seed=0 + X_SEED_OFFSET)
    return W, X


def gate_projection(seed: int = 1, N: int = 14336, K: int = 4096, std: float = 0.02):
    """Llama-3.1-8B-shaped gate/up projection W[14336, 4096] with 0.1% t_3 tail."""
    return weight_with_tail(N, K, seed=seed, std=std)


def down_projection(seed: int = 4, N: int = 4096, K: int = 14336, std: float = 0.02):
    """Llama-3.1-8B-shaped down projection W[4096, 14336] with 0.1% t_3 tail."""
    return weight_with_tail(N, K, seed=seed, std=std)


def stack_layer(layer: int):
    """Layer `layer` of the 32-layer stack: (gate, up, down) with that layer's std."""
    sd = float(layer_stds()[layer])
    base = 1000 + 3 * layer
    return (weight_with_tail(14336, 4096, base, sd),
            weight_with_tail(14336, 4096, base + 1, sd),
            weight_with_tail(4096, 14336, base + 2, sd))


# --------------------------------------------------------------------------
# Device-side draws for the benchmark's 32-layer stack (5.6 G weights): the
# same distributions as weight_with_tail, drawn with a CUDA torch.Generator
# so that generating the stack takes seconds instead of minutes.  The bits
# differ from the host recipe; anything that compares against the oracle
# copies the device bits back to the host first.
# --------------------------------------------------------------------------
def _gen_cuda(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight_with_tail_device(N: int, K: int, seed: int, device, std: float = 0.02, frac: float = 0.001) -> torch.Tensor:
    """Device BF16 W[N, K] ~ N(0, std) with a fraction `frac` of the elements
    (seeded distinct positions) replaced by std * t_3."""
    g = _gen_cuda(seed, device)
    w = torch.randn(N * K, generator=g, dtype=torch.float32, device=device) * std
    cnt = int(round(frac * N * K))
    if cnt:
        pos = torch.randperm(N * K, generator=g, device=device)[:cnt]
        z = torch.randn(cnt, generator=g, dtype=torch.float64, device=device)
        c = torch.randn(3, cnt, generator=g, dtype=torch.float64, device=device).pow(2).sum(0)
        w[pos] = std * (z / torch.sqrt(c / 3.0)).to(torch.float32)
    return w.view(N, K).to(torch.bfloat16)


def stack_layer_device(layer: int, device):
    """Layer `layer` of the 32-layer stack drawn on the device: (gate, up,
    down) BF16 tensors with that layer's std, seeds 1000 + 3*layer (+0, +1, +2)."""
    sd = float(layer_stds()[layer])
    base = 1000 + 3 * layer
    return (weight_with_tail_device(14336, 4096, base, device, sd),
            weight_with_tail_device(14336, 4096, base + 1, device, sd),
            weight_with_tail_device(4096, 14336, base + 2, device, sd))


def activations_device(M: int, K: int, seed: int, device) -> torch.Tensor:
    """Device BF16 X[M, K] ~ N(0, 1)."""
    g = _gen_cuda(seed, device)
    return torch.randn(M, K, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)
