"""Fused activation quantization + scaled_mm (lq_quant_scaled_mm): the codes
and scales it writes are bit-exact against the oracle's quantizer, C is
within tolerance of the oracle, and C equals - bit for bit - the two-step
path (lq_quant_per_token, then lq_scaled_mm with the same variant)."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import FMT_NAME, assert_close

pytestmark = pytest.mark.gpu

SHAPES = [(1, 384, 1152), (5, 256, 1040), (16, 512, 4096), (24, 384, 2048), (32, 256, 1152), (40, 256, 1024)]
VARIANTS = [dict(swap_ab=1, tile_n=16, split_k=1, stages=2), dict(swap_ab=1, tile_n=16, split_k=8, stages=2),
            dict(swap_ab=1, tile_n=32, split_k=4, stages=3), dict(swap_ab=1, tile_n=64, split_k=2, stages=2),
            dict(swap_ab=1, tile_n=32, split_k=16, stages=2)]


def _vid(v):
    return f"tn{v['tile_n']}-s{v['split_k']}"


@pytest.fixture
def always_fuse():
    """Every fusable variant takes the one-kernel path, whatever its slice."""
    old = lq.set_fuse_limit(1 << 40)
    yield
    lq.set_fuse_limit(-1)
    assert old == lq.set_fuse_limit(-1)


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8], ids=["fp8", "int8"])
@pytest.mark.parametrize("vd", VARIANTS, ids=_vid)
def test_fused_matches_oracle_and_two_step(cuda_device, always_fuse, fmt, vd):
    name = FMT_NAME[fmt]
    for (M, N, K) in SHAPES:
        if vd["split_k"] * vd["tile_n"] > 512:
            continue
        x = inputs.activations(M, K, seed=inputs.stable_seed("fused-A", M, N, K))
        w = inputs.weights(N, K, seed=inputs.stable_seed("fused-W", N, K)).float().numpy()
        qb, sb = O.quant_per_channel(w, name)
        B = torch.from_numpy(qb).cuda()
        b_s = torch.from_numpy(sb).cuda()
        v = lq.make_variant(reduce=2, **vd)
        C, q, s = lq.quant_scaled_mm(fmt, x.cuda(), B, b_s, variant=v)
        torch.cuda.synchronize()
        assert lq.device_status(0) == 0
        ra, rsa = O.quant_per_token(x.float().numpy(), name)
        assert np.array_equal(s.cpu().numpy(), rsa), (M, N, K)
        assert np.array_equal(q.cpu().numpy(), ra), (M, N, K)
        assert_close(C, O.scaled_mm_ref(name, ra, rsa, qb, sb), f"fused M={M} N={N} K={K} {vd}")
        q2, s2 = lq.quant_per_token(fmt, x.cuda())
        C2 = lq.scaled_mm(fmt, q2, s2, B, b_s, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(C, C2), (M, N, K)


def test_fused_default_variant_and_fallback(cuda_device):
    """variant = NULL (table / heuristic) and a Standard variant (two-kernel
    fallback) give the same codes and C as the two-step path."""
    M, N, K = 8, 1024, 4096
    x = inputs.activations(M, K, seed=7).cuda()
    w = inputs.weights(N, K, seed=8).cuda()
    for fmt in ("fp8_dynamic", "w8a8_int8"):
        qb, sb = lq.quant_per_token(fmt, w)
        for v in (None, lq.make_variant(swap_ab=0, tile_n=128, split_k=2, stages=3, reduce=2)):
            C, q, s = lq.quant_scaled_mm(fmt, x, qb, sb, variant=v)
            q2, s2 = lq.quant_per_token(fmt, x)
            C2 = lq.scaled_mm(fmt, q2, s2, qb, sb, variant=v)
            torch.cuda.synchronize()
            assert torch.equal(q, q2) and torch.equal(s, s2) and torch.equal(C, C2)


@pytest.mark.parametrize("limit", [-1, 1 << 40], ids=["default-limit", "always-fuse"])
def test_fused_qwen_shapes_against_two_step(cuda_device, limit):
    """Full decode shapes with the table's variants, with the default fusion
    limit and with every fusable variant fused."""
    lq.set_fuse_limit(limit)
    try:
        _qwen_shapes()
    finally:
        lq.set_fuse_limit(-1)


def _qwen_shapes():
    for (K, N) in inputs.QWEN3_8B.values():
        for M in (1, 16, 32):
            x = inputs.activations(M, K, seed=M + K).cuda()
            w = inputs.weights(N, K, seed=N + K).cuda()
            qb, sb = lq.quant_per_token("fp8_dynamic", w)
            C, q, s = lq.quant_scaled_mm("fp8_dynamic", x, qb, sb)
            q2, s2 = lq.quant_per_token("fp8_dynamic", x)
            C2 = lq.scaled_mm("fp8_dynamic", q2, s2, qb, sb)
            torch.cuda.synchronize()
            assert torch.equal(q, q2) and torch.equal(s, s2)
            assert torch.equal(C, C2), (M, N, K)


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
def test_fused_wide_range_rows(cuda_device, always_fuse, fmt):
    """Tokens whose scales take both ways of dividing (around amax = 2^-80,
    subnormal elements, scales near the top of fp32): the fused kernel's
    codes and scales are still the oracle's, C the two-step path's."""
    from _lqtest import wide_range_rows
    K, N = 1024, 256
    x = wide_range_rows(K, seed=11).cuda()
    M = x.shape[0]
    w = inputs.weights(N, K, seed=12).cuda()
    qb, sb = lq.quant_per_token(fmt, w)
    for vd in (dict(swap_ab=1, tile_n=16, split_k=1, stages=2), dict(swap_ab=1, tile_n=16, split_k=4, stages=2)):
        v = lq.make_variant(reduce=2, **vd)
        C, q, s = lq.quant_scaled_mm(fmt, x, qb, sb, variant=v)
        torch.cuda.synchronize()
        ra, rsa = O.quant_per_token(x.float().cpu().numpy(), fmt)
        assert np.array_equal(s.cpu().numpy(), rsa)
        assert np.array_equal(q.cpu().numpy(), ra)
        C2 = lq.scaled_mm(fmt, q, s, qb, sb, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(C, C2)
