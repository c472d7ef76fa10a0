"""GPU parity of the quantizer kernels: codes and scales bit-exact against the
oracle on the same bf16 inputs (called through the C ABI)."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import wide_range_rows

pytestmark = pytest.mark.gpu

PER_TOKEN_SHAPES = [(1, 16), (3, 128), (16, 2048), (32, 4096), (7, 4112), (24, 12288), (64, 25600), (300, 1024), (2, 40960), (5, 2064)]


def _x(M, K, seed, outliers=True):
    return inputs.activations(M, K, seed=seed, outliers=outliers)


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
@pytest.mark.parametrize("M,K", PER_TOKEN_SHAPES)
def test_quant_per_token_bitexact(cuda_device, fmt, M, K):
    x = _x(M, K, seed=M * 7919 + K)
    q, s = lq.quant_per_token(fmt, x.to(cuda_device))
    torch.cuda.synchronize()
    q_ref, s_ref = O.quant_per_token(x.float().numpy(), fmt)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    if fmt == "w8a8_int8":
        assert np.array_equal(q.cpu().numpy(), q_ref)
    else:
        assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
def test_quant_per_token_special_rows(cuda_device, fmt):
    """Zero rows (scale floor), a row with a negative zero, ties, saturation edge."""
    x = torch.zeros((5, 256), dtype=torch.float32)
    x[1, 0] = -0.0
    x[1, 1] = 1e-30          # tiny: scale below the floor before clamping
    x[2, :] = torch.linspace(-3, 3, 256)
    x[3, 0], x[3, 1], x[3, 2] = 448.0, 1.0625 * 0 + 232.0, -0.5
    x[4, :] = 1.0            # all equal: every code hits Q
    xb = x.to(torch.bfloat16)
    q, s = lq.quant_per_token(fmt, xb.to(cuda_device))
    q_ref, s_ref = O.quant_per_token(xb.float().numpy(), fmt)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
@pytest.mark.parametrize("K", [256, 4096, 12288])
def test_quant_per_token_wide_range_rows(cuda_device, fmt, K):
    xb = wide_range_rows(K, seed=K)
    q, s = lq.quant_per_token(fmt, xb.to(cuda_device))
    q_ref, s_ref = O.quant_per_token(xb.float().numpy(), fmt)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_group128_wide_range_rows(cuda_device):
    xb = wide_range_rows(1024, seed=3)
    # every 128-group of a row spans a different slice of the exponent range
    q, s = lq.quant_per_token_group128(xb.to(cuda_device))
    q_ref, s_ref = O.quant_per_token_group128(xb.float().numpy())
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("M,K", [(1, 128), (5, 384), (32, 5120), (3, 25600), (257, 1024)])
def test_quant_group128_bitexact(cuda_device, M, K):
    x = _x(M, K, seed=M * 131 + K)
    q, s = lq.quant_per_token_group128(x.to(cuda_device))
    q_ref, s_ref = O.quant_per_token_group128(x.float().numpy())
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (1024, 2048)])
def test_quant_weight_block128_bitexact(cuda_device, N, K):
    w = inputs.weights(N, K, seed=N + K)
    q, s = lq.quant_weight_block128(w.to(cuda_device))
    q_ref, s_ref = O.quant_weight_block128(w.float().numpy())
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_per_channel_weight_is_per_token_call(cuda_device):
    w = inputs.weights(512, 1024, seed=5)
    q, s = lq.quant_per_token("fp8_dynamic", w.to(cuda_device))
    q_ref, s_ref = O.quant_per_channel(w.float().numpy(), "fp8_dynamic")
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_empty_is_noop(cuda_device):
    x = torch.empty((0, 128), dtype=torch.bfloat16, device=cuda_device)
    q, s = lq.quant_per_token("fp8_dynamic", x)
    assert q.shape == (0, 128) and s.shape == (0,)
