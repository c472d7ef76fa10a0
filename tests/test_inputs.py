"""The seeded input recipe shared by the tests, the benchmark and the oracle
checks: deterministic for a seed, the documented distributions, the outlier
channels and the synthetic router's invariants.  CPU only."""

import math

import numpy as np
import torch

from quantized_linear_gemm_b200 import inputs


def test_same_seed_same_tensor_and_stable_seeds():
    a = inputs.activations(8, 512, seed=5)
    assert torch.equal(a, inputs.activations(8, 512, seed=5))
    assert not torch.equal(a, inputs.activations(8, 512, seed=6))
    assert torch.equal(inputs.weights(64, 256, seed=1), inputs.weights(64, 256, seed=1))
    assert inputs.stable_seed("A", 0, 8, 4096) == inputs.stable_seed("A", 0, 8, 4096)
    assert inputs.stable_seed("A", 0, 8, 4096) != inputs.stable_seed("A", 0, 8, 4097)
    assert 0 <= inputs.stable_seed("x") < 2 ** 32


def test_activation_recipe():
    """N(0, 1) with ceil(1% of K) outlier channels scaled by 20, in bf16."""
    M, K = 512, 4096
    x = inputs.activations(M, K, seed=3)
    assert x.dtype == torch.bfloat16 and x.shape == (M, K)
    std = x.float().std(dim=0)
    out = std > 5
    assert int(out.sum()) == math.ceil(0.01 * K)
    assert abs(float(std[out].mean()) - 20) < 2 and abs(float(std[~out].mean()) - 1) < 0.05
    plain = inputs.activations(M, K, seed=3, outliers=False).float()
    assert float(plain.std(dim=0).max()) < 1.5
    assert abs(float(plain.mean())) < 0.01


def test_weight_recipe():
    w = inputs.weights(1024, 1024, seed=2)
    assert w.dtype == torch.bfloat16 and w.shape == (1024, 1024)
    assert abs(float(w.float().std()) - 0.02) < 5e-4 and abs(float(w.float().mean())) < 5e-4


def test_router_counts():
    """Each token picks top_k distinct experts: the counts sum to tokens x
    top_k, no expert gets more than `tokens`, and the draw is seeded."""
    E, k = inputs.QWEN3_30B_A3B_NUM_EXPERTS, inputs.QWEN3_30B_A3B_TOP_K
    for tokens in (1, 8, 64):
        c = inputs.expert_counts(tokens, E, k, seed=tokens)
        assert c.shape == (E,) and c.dtype == np.int64
        assert int(c.sum()) == tokens * k and int(c.max()) <= tokens and int(c.min()) >= 0
        assert np.array_equal(c, inputs.expert_counts(tokens, E, k, seed=tokens))
    assert int((inputs.expert_counts(1, E, k, seed=0) > 0).sum()) == k   # one token: k distinct experts
