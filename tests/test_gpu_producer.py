"""GPU parity of the producer-side fused quantizers (RMSNorm or
SiLU-and-multiply, then per-token or 1 x 128 quantization), called through
the C ABI: codes and scales bit-exact against the oracle, the updated
residual equal to the oracle's, on seeded inputs of the Qwen3 shapes, ragged
and maximal rows, and rows that stress the rounding paths."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from oracle import producer_oracle as P
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import wide_range_rows

pytestmark = pytest.mark.gpu

FMTS = ["fp8_dynamic", "w8a8_int8"]
# (M, K): decode and prefill rows of Qwen3-8B / 32B hidden sizes, a ragged
# count of rows, a short row, and the longest row a CTA holds.
RMS_SHAPES = [(1, 4096), (5, 5120), (32, 4096), (300, 1024), (7, 144), (2, 32768), (3, 128),
              (400, 5120), (296, 32768)]   # >= 296 rows: persistent CTAs with rows staged in shared memory
# (M, I): Qwen3-8B / 32B intermediate sizes, ragged, short, longest.
SILU_SHAPES = [(1, 12288), (8, 25600), (33, 1024), (4, 144), (2, 32768), (64, 128),
               (300, 1024), (333, 25600), (296, 12288), (301, 32768)]   # staged, at the size limit, too long


def _np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _weight(K, seed):
    g = torch.Generator().manual_seed(seed)
    return (1.0 + 0.1 * torch.randn(K, generator=g)).to(torch.bfloat16)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,K", RMS_SHAPES)
@pytest.mark.parametrize("with_residual", [False, True], ids=["plain", "residual"])
def test_rms_norm_dynamic_per_token_quant(cuda_device, fmt, M, K, with_residual):
    x = inputs.activations(M, K, seed=inputs.stable_seed("rms-x", M, K))
    w = _weight(K, K)
    res = inputs.activations(M, K, seed=inputs.stable_seed("rms-r", M, K)) if with_residual else None
    res_d = res.cuda() if res is not None else None
    q, s = lq.rms_norm_dynamic_per_token_quant(fmt, x.cuda(), w.cuda(), 1e-6, residual=res_d)
    torch.cuda.synchronize()
    q_ref, s_ref, h_ref = P.rms_norm_dynamic_per_token_quant(_np(x), _np(w), 1e-6, fmt,
                                                             residual=None if res is None else _np(res))
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    if res_d is not None:
        assert np.array_equal(_np(res_d), h_ref)


@pytest.mark.parametrize("M,K", [(1, 4096), (5, 5120), (32, 4096), (257, 1024), (2, 32768), (3, 128), (310, 4096)])
@pytest.mark.parametrize("with_residual", [False, True], ids=["plain", "residual"])
def test_rms_norm_per_block_quant(cuda_device, M, K, with_residual):
    x = inputs.activations(M, K, seed=inputs.stable_seed("rmsb-x", M, K))
    w = _weight(K, K + 1)
    res = inputs.activations(M, K, seed=inputs.stable_seed("rmsb-r", M, K)) if with_residual else None
    res_d = res.cuda() if res is not None else None
    q, s = lq.rms_norm_per_block_quant(x.cuda(), w.cuda(), 1e-5, residual=res_d)
    torch.cuda.synchronize()
    q_ref, s_ref, h_ref = P.rms_norm_per_block_quant(_np(x), _np(w), 1e-5, residual=None if res is None else _np(res))
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    if res_d is not None:
        assert np.array_equal(_np(res_d), h_ref)


def _gate_up(M, I, seed):
    g = inputs.activations(M, I, seed=seed).float() * 2
    u = inputs.activations(M, I, seed=seed + 1)
    return torch.cat([g.to(torch.bfloat16), u], dim=1)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("M,I", SILU_SHAPES)
def test_silu_and_mul_dynamic_per_token_quant(cuda_device, fmt, M, I):
    gu = _gate_up(M, I, seed=inputs.stable_seed("silu", M, I))
    q, s = lq.silu_and_mul_dynamic_per_token_quant(fmt, gu.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = P.silu_and_mul_dynamic_per_token_quant(_np(gu), fmt)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("M,I", [(1, 12288), (8, 25600), (33, 1024), (2, 32768), (64, 128), (300, 12288),
                                 (297, 128)])
def test_silu_and_mul_per_block_quant(cuda_device, M, I):
    gu = _gate_up(M, I, seed=inputs.stable_seed("silub", M, I))
    q, s = lq.silu_and_mul_per_block_quant(gu.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = P.silu_and_mul_per_block_quant(_np(gu))
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_silu_rounding_paths(cuda_device):
    """Every bf16 value as the gate (both signs, subnormals, the fp64 region
    g <= -80, the overflow of exp in fp32 near -89, +-0, huge), times u = 1 and
    u = 3: the SiLU is rounded once from its exact value on both sides."""
    bits = torch.arange(1 << 16, dtype=torch.int32)
    g = (bits << 16).view(torch.float32)
    g = g[torch.isfinite(g)]                       # 65280 finite bf16 values = 51 rows of 1280
    g = g.to(torch.bfloat16).reshape(-1, 1280)
    for uval in (1.0, 0.375):                      # no product overflows bf16
        u = torch.full_like(g, uval)
        gu = torch.cat([g, u], dim=1)
        for fmt in FMTS:
            q, s = lq.silu_and_mul_dynamic_per_token_quant(fmt, gu.cuda())
            torch.cuda.synchronize()
            q_ref, s_ref = P.silu_and_mul_dynamic_per_token_quant(_np(gu), fmt)
            assert np.array_equal(s.cpu().numpy(), s_ref), (fmt, uval)
            assert np.array_equal(q.cpu().numpy(), q_ref), (fmt, uval)
        # one scale per 128 values: many more codes sit next to their group's amax
        q, s = lq.silu_and_mul_per_block_quant(gu.cuda())
        torch.cuda.synchronize()
        q_ref, s_ref = P.silu_and_mul_per_block_quant(_np(gu))
        assert np.array_equal(s.cpu().numpy(), s_ref), uval
        assert np.array_equal(q.cpu().numpy(), q_ref), uval


def test_silu_bf16_every_gate(cuda_device):
    """The producer kernels' SiLU (all of its tiers, through the test hook)
    on every finite bf16 gate: bf16(silu(g)) bit for bit equal to the
    oracle's value rounded once from the exact quotient.  Codes can hide a
    wrong last bit of the SiLU; this compares the SiLU itself."""
    bits = torch.arange(1 << 16, dtype=torch.int32)
    g = (bits << 16).view(torch.float32)
    g = g[torch.isfinite(g)].to(torch.bfloat16)
    out = lq.test_silu_bf16(g.cuda())
    torch.cuda.synchronize()
    ref = P.silu_bf16(g.double().numpy())
    got = out.double().cpu().numpy()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), (g[~torch.from_numpy(same)][:8], got[~same][:8], ref[~same][:8])
    # the same gates again in another order (the kernel's grid-stride loop splits them differently)
    perm = torch.randperm(g.numel(), generator=torch.Generator().manual_seed(7))
    out2 = lq.test_silu_bf16(g[perm].contiguous().cuda())
    torch.cuda.synchronize()
    assert torch.equal(out2.cpu(), out.cpu()[perm])


def test_silu_ties_of_tiny_gates(cuda_device):
    """Gates 0 < |g| < 2^-125 where g / 2 lies halfway between two bf16
    values (odd multiples of 2^-133, both signs), alone in a row so that the
    scale floor 2^-126 makes their codes depend on the silu's last bit: the
    silu goes towards +inf at those ties (silu(g) > g / 2), codes bit-exact
    against the oracle.  u = 3.984375 makes 40 of the FP8 codes differ from
    those of a silu rounded ties-to-even."""
    k = torch.arange(1, 256, 2, dtype=torch.float64)
    mag = k * 2.0 ** -133
    g = torch.cat([mag, -mag]).to(torch.float32).to(torch.bfloat16)[None, :]   # 256 gates, exact in bf16
    assert torch.equal(g.double()[0, :128], mag)
    for uval in (1.0, 3.984375):
        gu = torch.cat([g, torch.full_like(g, uval)], dim=1)
        for fmt in FMTS:
            q, s = lq.silu_and_mul_dynamic_per_token_quant(fmt, gu.cuda())
            torch.cuda.synchronize()
            q_ref, s_ref = P.silu_and_mul_dynamic_per_token_quant(_np(gu), fmt)
            assert np.array_equal(s.cpu().numpy(), s_ref), (fmt, uval)
            assert np.array_equal(q.cpu().numpy(), q_ref), (fmt, uval)
        q, s = lq.silu_and_mul_per_block_quant(gu.cuda())
        torch.cuda.synchronize()
        q_ref, s_ref = P.silu_and_mul_per_block_quant(_np(gu))
        assert np.array_equal(s.cpu().numpy(), s_ref), uval
        assert np.array_equal(q.cpu().numpy(), q_ref), uval


@pytest.mark.parametrize("fmt", FMTS)
def test_rms_norm_wide_range_rows(cuda_device, fmt):
    """Rows spanning 230 binades, subnormal entries, amax around 2^-80 (both
    ways of dividing by the scale), with a large eps and with eps = 0."""
    x = wide_range_rows(4096, seed=21)
    w = _weight(4096, 22)
    for eps in (0.0, 1e-6, 4.0):
        q, s = lq.rms_norm_dynamic_per_token_quant(fmt, x.cuda(), w.cuda(), eps)
        torch.cuda.synchronize()
        q_ref, s_ref, _ = P.rms_norm_dynamic_per_token_quant(_np(x), _np(w), eps, fmt)
        assert np.array_equal(s.cpu().numpy(), s_ref), eps
        assert np.array_equal(q.cpu().numpy(), q_ref), eps


def test_rms_norm_zero_rows_and_equal_rows(cuda_device):
    K = 1024
    x = torch.zeros((3, K), dtype=torch.bfloat16)
    x[1, :] = 2.0 ** -20
    x[2, :] = -3.0
    w = _weight(K, 23)
    for fmt in FMTS:
        q, s = lq.rms_norm_dynamic_per_token_quant(fmt, x.cuda(), w.cuda(), 1e-6)
        torch.cuda.synchronize()
        q_ref, s_ref, _ = P.rms_norm_dynamic_per_token_quant(_np(x), _np(w), 1e-6, fmt)
        assert np.array_equal(s.cpu().numpy(), s_ref)
        assert np.array_equal(q.cpu().numpy(), q_ref)


def test_producer_quant_feeds_scaled_mm(cuda_device):
    """The codes and scales go straight into lq_scaled_mm: C is within the
    suite's tolerance of the oracle's product of the oracle's codes."""
    M, K, N = 8, 4096, 1024
    x = inputs.activations(M, K, seed=31)
    w_norm = _weight(K, 32)
    wq = inputs.weights(N, K, seed=33).float().numpy()
    qb, sb = O.quant_per_channel(wq, "fp8_dynamic")
    q, s = lq.rms_norm_dynamic_per_token_quant("fp8_dynamic", x.cuda(), w_norm.cuda(), 1e-6)
    C = lq.scaled_mm("fp8_dynamic", q, s, torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda())
    torch.cuda.synchronize()
    q_ref, s_ref, _ = P.rms_norm_dynamic_per_token_quant(_np(x), _np(w_norm), 1e-6, "fp8_dynamic")
    ok, worst = O.within_tolerance(_np(C), O.scaled_mm_ref("fp8_dynamic", q_ref, s_ref, qb, sb))
    assert ok, worst


def test_producer_empty_is_noop(cuda_device):
    x = torch.empty((0, 128), dtype=torch.bfloat16, device=cuda_device)
    q, s = lq.rms_norm_dynamic_per_token_quant("fp8_dynamic", x, torch.ones(128, dtype=torch.bfloat16,
                                                                             device=cuda_device), 1e-6)
    assert q.shape == (0, 128) and s.shape == (0,)
    q, s = lq.silu_and_mul_per_block_quant(torch.empty((0, 256), dtype=torch.bfloat16, device=cuda_device))
    assert q.shape == (0, 128) and s.shape == (0, 1)


def test_staged_rows_leave_the_status_word_clear(cuda_device):
    """The persistent kernels wait (bounded) for their row copies; a normal
    run leaves no timeout bit set."""
    assert lq.device_status(0) == 0
    gu = _gate_up(600, 4096, seed=41).cuda()
    lq.silu_and_mul_dynamic_per_token_quant("fp8_dynamic", gu)
    x = inputs.activations(600, 4096, seed=42).cuda()
    lq.rms_norm_per_block_quant(x, torch.ones(4096, dtype=torch.bfloat16, device="cuda"), 1e-6,
                                residual=torch.zeros_like(x))
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
