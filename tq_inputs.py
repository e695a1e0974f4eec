"""Seeded synthetic inputs for the weight-only low-bit linear layer.

This module only draws random numbers and shapes; it holds none of the method's arithmetic
(no thresholds, codes, scales or products), so both the CUDA path and the CPU oracle can be fed
from it without sharing any of the computation.

Workloads (no trained checkpoints exist here, so random-init tensors of the real shapes stand in
for them; no public benchmark suite is involved):
  * weights  W ~ N(0, 0.02) fp32 (optionally a fraction of entries multiplied by 10, seeded
    positions), one distinct matrix per (config, layer, matrix) seed;
  * decode activations x ~ N(0, 1) fp16;
  * prefill activations x ~ N(0, 1) fp16 with 1 % of the rows (seeded permutation) times 20;
  * bias ~ N(0, 0.01) fp16.
Seeds: seed = 1000 * config + 16 * layer + matrix_id.
"""
from __future__ import annotations

import torch

# Linear shapes (N = out features, K = in features) of the two model families.
LLAMA3_8B = {
    "q_proj": (4096, 4096),
    "k_proj": (1024, 4096),
    "v_proj": (1024, 4096),
    "o_proj": (4096, 4096),
    "gate_proj": (14336, 4096),
    "up_proj": (14336, 4096),
    "down_proj": (4096, 14336),
}
LLAMA3_8B_LAYERS = 32

QWEN2_7B = {
    "qkv_proj": (4608, 3584),
    "o_proj": (3584, 3584),
    "gate_up_proj": (37888, 3584),
    "down_proj": (3584, 18944),
}
QWEN2_7B_LAYERS = 28


def seed_for(config: int, layer: int, matrix_id: int) -> int:
    return 1000 * config + 16 * layer + matrix_id


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, seed: int, device="cpu", sigma: float = 0.02,
            outlier_frac: float = 0.0, outlier_mult: float = 10.0,
            dtype=torch.float32) -> torch.Tensor:
    """W[N,K] ~ N(0, sigma), a seeded `outlier_frac` of entries multiplied by `outlier_mult`."""
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * sigma
    if outlier_frac > 0:
        n_out = max(1, int(round(outlier_frac * N * K)))
        idx = torch.randint(0, N * K, (n_out,), generator=g, device=device)
        w.view(-1)[idx] *= outlier_mult
    return w.to(dtype)


def activations(M: int, K: int, seed: int, device="cpu", outlier_row_frac: float = 0.0,
                outlier_mult: float = 20.0) -> torch.Tensor:
    """x[M,K] ~ N(0,1) fp16; a seeded `outlier_row_frac` of the rows multiplied by `outlier_mult`."""
    g = _gen(seed + 7919, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if outlier_row_frac > 0 and M > 0:
        n_out = max(1, int(round(outlier_row_frac * M)))
        rows = torch.randperm(M, generator=g, device=device)[:n_out]
        x[rows] *= outlier_mult
    return x.to(torch.float16)


def bias(N: int, seed: int, device="cpu", sigma: float = 0.01) -> torch.Tensor:
    g = _gen(seed + 104729, device)
    return (torch.randn(N, generator=g, device=device, dtype=torch.float32) * sigma).to(torch.float16)


def random_codes(N: int, K: int, seed: int, device="cpu", probs=(1 / 3, 1 / 3, 1 / 3)) -> torch.Tensor:
    """Random ternary code indices in {0,1,2} (for tests that start from codes, not weights)."""
    g = _gen(seed, device)
    p = torch.tensor(probs, dtype=torch.float64, device=device)
    return torch.multinomial(p, N * K, replacement=True, generator=g).view(N, K).to(torch.uint8)


def small_int_activations(M: int, K: int, seed: int, lo: int = -4, hi: int = 4, device="cpu") -> torch.Tensor:
    """Integer-valued fp16 activations in [lo, hi] (products and sums stay exact in fp32/fp64)."""
    g = _gen(seed, device)
    return torch.randint(lo, hi + 1, (M, K), generator=g, device=device).to(torch.float16)
