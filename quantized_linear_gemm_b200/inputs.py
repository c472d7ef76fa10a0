"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module only draws random bf16 tensors of the shapes the workloads use.
It holds none of the GEMM's or the quantizers' arithmetic, so that both the
CUDA path and the CPU oracle can consume the same inputs without sharing any
of the method's code.

Workloads (all synthetic; no dataset is involved):

* activations A[M, K]: N(0, 1) in fp32, with ceil(1% of K) channels, chosen
  by the generator, multiplied by 20 (outlier channels), rounded to bf16;
* weights W[N, K] (linear-layer layout, output channel major): N(0, 0.02),
  rounded to bf16.

Shapes are Qwen3 decoder linears (K = in_features, N = out_features).
"""

from __future__ import annotations

import hashlib

import numpy as np

import torch

# (K, N) of the four linears of a Qwen3 decoder layer
QWEN3_8B = {
    "qkv": (4096, 6144),
    "o": (4096, 4096),
    "gate_up": (4096, 24576),
    "down": (12288, 4096),
}
QWEN3_32B = {
    "qkv": (5120, 10240),
    "o": (8192, 5120),
    "gate_up": (5120, 51200),
    "down": (25600, 5120),
}
DECODE_M = (1, 2, 4, 8, 16, 24, 32)
PREFILL_M = (256, 2048, 8192)


def stable_seed(*parts) -> int:
    """A seed that depends only on the given labels (stable across runs/hosts)."""
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:4], "little")


def activations(M: int, K: int, seed: int, outliers: bool = True,
                outlier_frac: float = 0.01, outlier_gain: float = 20.0) -> torch.Tensor:
    """bf16 [M, K] on the CPU: N(0,1), optionally with outlier channels."""
    g = torch.Generator().manual_seed(int(seed))
    x = torch.randn((M, K), generator=g, dtype=torch.float32)
    if outliers and K > 0:
        n_out = -(-int(round(outlier_frac * K * 1000)) // 1000)  # ceil(frac * K)
        n_out = max(1, min(K, n_out))
        cols = torch.randperm(K, generator=g)[:n_out]
        x[:, cols] *= outlier_gain
    return x.to(torch.bfloat16)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """bf16 [N, K] on the CPU: N(0, std)."""
    g = torch.Generator().manual_seed(int(seed))
    w = torch.randn((N, K), generator=g, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def uniform_codes(shape, seed: int, lo: int, hi: int) -> torch.Tensor:
    """Uniform random integers in [lo, hi) as int64 (raw operand bytes for edge tests)."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randint(lo, hi, tuple(shape), generator=g, dtype=torch.int64)


# Mixture-of-experts decode (Qwen3-30B-A3B sizes: 128 experts, 8 chosen per
# token, hidden 2048, expert intermediate 768): (K, N) of the two expert GEMMs.
QWEN3_30B_A3B_EXPERTS = {"gate_up": (2048, 1536), "down": (768, 2048)}
QWEN3_30B_A3B_NUM_EXPERTS = 128
QWEN3_30B_A3B_TOP_K = 8


def expert_counts(tokens: int, num_experts: int, top_k: int, seed: int) -> np.ndarray:
    """Tokens routed to each expert when each of `tokens` tokens picks
    `top_k` distinct experts uniformly at random (a seeded stand-in for a
    router).  int64 [num_experts]."""
    g = np.random.default_rng(seed)
    counts = np.zeros(num_experts, dtype=np.int64)
    for _ in range(tokens):
        counts[g.choice(num_experts, size=top_k, replace=False)] += 1
    return counts
