"""Seeded synthetic inputs shaped like the pages' models.

This module draws random numbers and names shapes; it holds none of the method's
arithmetic (no absmean, no rounding, no quantisation).  It is the one module that both
the CUDA path's callers (tests, benchmark) and the CPU oracle's callers use, so that
both sides see the same bytes.

Workloads (``nn.Linear`` convention: W is [N = out, K = in], X is [M, K]):
  * toy  -- BitLinear 256 -> 512, the FFN up-projection of the 6-layer, hidden-256,
            FFN-512 model trained in "Which 1-Bit Weights Can You Trust?"
            (section "Experimental Setup"); 32 sequences x 256 tokens.
  * llama700m / llama3b / llama70b -- the seven BitLinear projections of one layer of
            the LLaMA-shaped models that "1.58 bits: what BitNet promised and what it
            required" (section "The parity claim, with its numbers") and
            "1-bit & Ternary LLMs" (section "Reported results") compare.
  * sweep -- square and rectangular ternary GEMMs.

Distributions: W ~ N(0, sigma) fp32 (sigma = 0.02); optionally a fraction of entries
drawn from N(0, 1e-3 sigma) to raise the share of zero codes (absmean is scale
invariant, so scaling sigma alone cannot change that share).  X is bf16 of N(0, 1)
with round(f K) (at least one) outlier channels multiplied by a constant.
"""
from __future__ import annotations

import torch

SIGMA = 0.02


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def weight(N: int, K: int, seed: int, sigma: float = SIGMA, small_frac: float = 0.0,
           small_scale: float = 1e-3) -> torch.Tensor:
    """fp32 [N, K] weight matrix on the CPU."""
    g = _gen(seed)
    W = torch.randn(N, K, generator=g, dtype=torch.float32) * sigma
    if small_frac > 0.0:
        pick = torch.rand(N, K, generator=g) < small_frac
        W = torch.where(pick, W * small_scale, W)
    return W


def activations(M: int, K: int, seed: int, outlier_frac: float = 0.01,
                outlier_scale: float = 20.0) -> torch.Tensor:
    """bf16 [M, K] activations on the CPU with heavy-tailed outlier channels."""
    g = _gen(seed + 1_000_003)
    X = torch.randn(M, K, generator=g, dtype=torch.float32)
    n_out = max(1, int(round(outlier_frac * K)))
    cols = torch.randperm(K, generator=g)[:n_out]
    X[:, cols] *= outlier_scale
    return X.to(torch.bfloat16)


def codes(N: int, K: int, seed: int, p_zero: float = 0.31) -> torch.Tensor:
    """int8 [N, K] ternary codes drawn directly (for the pack entry point)."""
    g = _gen(seed + 2_000_003)
    u = torch.rand(N, K, generator=g)
    c = torch.where(u < p_zero, 0, torch.where(u < p_zero + (1 - p_zero) / 2, 1, -1))
    return c.to(torch.int8)


def bf16_bits(X: torch.Tensor):
    """Raw uint16 bit patterns of a bf16 CPU tensor, as a numpy array."""
    import numpy as np
    return X.contiguous().view(torch.int16).numpy().view(np.uint16)


# Seven projections of one transformer layer: (name, N = out, K = in).
def layer_projections(hidden: int, ffn: int, kv_dim: int | None = None):
    kv = hidden if kv_dim is None else kv_dim
    return [("q", hidden, hidden), ("k", kv, hidden), ("v", kv, hidden), ("o", hidden, hidden),
            ("up", ffn, hidden), ("gate", ffn, hidden), ("down", hidden, ffn)]


WORKLOADS = {
    "toy": {"proj": [("up", 512, 256)], "M": [32 * 256], "outlier_frac": 0.005},
    "llama700m": {"proj": layer_projections(1536, 4096), "M": [1, 8, 512, 4096],
                  "outlier_frac": 0.01},
    "llama3b": {"proj": layer_projections(3200, 8640), "M": [1, 16, 2048, 8192],
                "outlier_frac": 0.01},
    "llama70b": {"proj": layer_projections(8192, 28672, kv_dim=1024),
                 "M": [1, 2, 4, 8, 16, 32, 64], "outlier_frac": 0.01},
}

SWEEP_KN = [1024, 2048, 4096, 8192, 16384]
SWEEP_M = [1, 4, 16, 64, 256, 1024, 8192]
# Sweep weight mixtures, named by the share of zero codes they give: the fraction of
# entries drawn from N(0, 1e-3 sigma) (`small_frac` of weight()).  A plain Gaussian gives
# about 31% zeros; 0.378 and 0.664 were solved for 50% and 70%.
SWEEP_SMALL_FRAC = {30: 0.0, 50: 0.378, 70: 0.664}
# Sweep activations: outlier-channel fractions and their scale.
SWEEP_OUTLIER_FRACS = [0.001, 0.005, 0.01, 0.02]
SWEEP_OUTLIER_SCALE = 50.0
# The grid's default point: 50% zero codes, 1% outlier channels.
SWEEP_DEFAULT_ZEROS = 50
SWEEP_DEFAULT_OUTLIERS = 0.01
