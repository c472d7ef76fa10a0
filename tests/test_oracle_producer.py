"""Pins of the producer-side oracle (RMSNorm / SiLU-and-multiply before the
dynamic quantization) against things other than itself: torch's own bf16
cast and fp64 rms_norm / silu, closed forms, exact special cases and
composition invariants.  CPU only."""

import math
from decimal import Context, Decimal
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import lq_oracle as O
from oracle import producer_oracle as P


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy().astype(np.float64)


def _ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


# ----------------------------------------------------------------- bf16_round
def test_bf16_round_keeps_every_bf16_value():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v32 = (bits << 16).view(np.float32)
    keep = ~np.isnan(v32)
    v = v32[keep].astype(np.float64)
    assert np.array_equal(P.bf16_round(v), v)


def test_bf16_round_matches_torch_cast_of_fp32_values():
    """For fp32 inputs a single rounding to bf16 is torch's cast (an
    independent round-to-nearest-even implementation)."""
    g = np.random.default_rng(1)
    v = (g.standard_normal(200000) * np.exp2(g.integers(-130, 120, 200000))).astype(np.float32)
    v = v[np.isfinite(v)]
    want = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    assert np.array_equal(P.bf16_round(v.astype(np.float64)), want)


def test_bf16_round_ties_and_single_rounding():
    lo = np.array([1.0, 1.0 + 2 ** -7, 3.0, 2.0 ** -126, 2.0 ** -133 * 5])
    step = np.array([2 ** -7, 2 ** -7, 2 ** -6, 2 ** -133, 2 ** -133])
    mid = lo + step / 2
    # ties go to the neighbour with an even last bit
    assert np.array_equal(P.bf16_round(mid), np.array([1.0, 1.0 + 2 ** -6, 3.0, 2.0 ** -126, 2.0 ** -133 * 6]))
    # just above a tie: up, although an fp32 detour would land on the tie and go to even
    above = mid + mid * 2.0 ** -40
    assert np.array_equal(P.bf16_round(above), lo + step)
    assert np.array_equal(P.bf16_round(-above), -(lo + step))


def test_bf16_round_overflow_and_zero():
    big = P.BF16_MAX + 2.0 ** 127 * 2 ** -8     # max + half an ulp: overflows
    assert np.isinf(P.bf16_round(np.array([big]))[0])
    assert P.bf16_round(np.array([P.BF16_MAX + 2.0 ** 127 * 2 ** -9]))[0] == P.BF16_MAX
    z = P.bf16_round(np.array([0.0, -0.0, 2.0 ** -135, -(2.0 ** -135)]))
    assert np.array_equal(z, [0.0, 0.0, 0.0, 0.0]) and np.signbit(z[1]) and np.signbit(z[3])


# ----------------------------------------------------------------- RMSNorm
def _rows(M, K, seed):
    from quantized_linear_gemm_b200 import inputs
    return inputs.activations(M, K, seed=seed).float().numpy().astype(np.float64)


def test_rms_norm_power_of_two_rows_are_exact():
    """A constant row of +-2^k has rms 2^k: with eps = 0 every normalised value
    is +-1 and y is the weight itself, exactly."""
    K = 256
    w = _bf16(np.random.default_rng(2).standard_normal(K))
    x = np.stack([np.full(K, 2.0 ** k) * s for k, s in [(0, 1), (-20, -1), (30, 1), (-100, 1)]])
    y, h = P.rms_norm_ref(x, w, eps=0.0)
    assert np.array_equal(h, x)
    assert np.array_equal(y, np.sign(x) * w[None, :])


@pytest.mark.parametrize("K,eps", [(128, 1e-6), (4096, 1e-6), (5120, 1e-5), (4096, 0.5)])
def test_rms_norm_against_torch_fp64(K, eps):
    """Within two bf16 units in the last place of torch's fp64 rms_norm
    (three roundings separate the two)."""
    x = _rows(6, K, seed=K)
    w = _bf16(1.0 + 0.1 * np.random.default_rng(K).standard_normal(K))
    y, _ = P.rms_norm_ref(x, w, eps)
    t = F.rms_norm(torch.from_numpy(x), (K,), torch.from_numpy(w), eps=float(np.float32(eps))).numpy()
    assert np.all(np.abs(y - t) <= 2 * _ulp_bf16(t) + 1e-30)


@pytest.mark.parametrize("mistake", ["mean_over_k_minus_1", "no_eps", "no_weight", "sqrt_not_rsqrt"])
def test_rms_norm_torch_pin_catches_planted_mistakes(mistake):
    K, eps = 16, 0.25          # small K: the mean over K - 1 is 6% off
    x = _rows(4, K, seed=3) * 0.5
    w = _bf16(1.5 + 0.1 * np.random.default_rng(4).standard_normal(K))
    v = {"mean_over_k_minus_1": (x * x).sum(1) / (K - 1) + eps, "no_eps": (x * x).mean(1),
         "no_weight": (x * x).mean(1) + eps, "sqrt_not_rsqrt": (x * x).mean(1) + eps}[mistake]
    r = np.sqrt(v) if mistake == "sqrt_not_rsqrt" else 1 / np.sqrt(v)
    wrong = P.bf16_round(x * r[:, None] * (1.0 if mistake == "no_weight" else w[None, :]))
    t = F.rms_norm(torch.from_numpy(x), (K,), torch.from_numpy(w), eps=eps).numpy()
    assert not np.all(np.abs(wrong - t) <= 2 * _ulp_bf16(t) + 1e-30)


def test_rms_norm_residual_is_added_first():
    """h = x + residual (exact for these small integers) is the new residual,
    and y is the RMSNorm of h."""
    g = np.random.default_rng(5)
    x = g.integers(-50, 50, (3, 256)).astype(np.float64)
    res = g.integers(-50, 50, (3, 256)).astype(np.float64)
    w = _bf16(g.standard_normal(256))
    y, h = P.rms_norm_ref(x, w, 1e-6, residual=res)
    assert np.array_equal(h, x + res)
    y2, _ = P.rms_norm_ref(x + res, w, 1e-6)
    assert np.array_equal(y, y2)


def test_rms_norm_zero_row_with_eps():
    y, _ = P.rms_norm_ref(np.zeros((1, 128)), np.ones(128), eps=1e-6)
    assert np.array_equal(y, np.zeros((1, 128)))


def test_rms_norm_is_scale_invariant_by_powers_of_two():
    """With eps = 0, scaling a row by 2^k changes nothing (every step scales
    exactly)."""
    x = _rows(3, 1024, seed=6)
    w = _bf16(np.random.default_rng(6).standard_normal(1024))
    y, _ = P.rms_norm_ref(x, w, 0.0)
    for k in (-40, 17):
        y2, _ = P.rms_norm_ref(x * 2.0 ** k, w, 0.0)
        assert np.array_equal(y, y2)


# ----------------------------------------------------------------- SiLU-and-multiply
def test_silu_and_mul_closed_forms():
    I = 8
    g = np.array([[0.0, 64.0, -64.0, 1e30, -1e30, 128.0, 256.0, -0.0]])
    u = np.array([[3.0, 0.5, 1.0, 2.0, 2.0, 0.25, 1.0, 5.0]])
    y = P.silu_and_mul_ref(np.concatenate([g, u], axis=1))
    assert y[0, 0] == 0.0
    assert y[0, 1] == 32.0                      # silu(64) rounds to 64 in bf16
    assert abs(y[0, 2]) < 1e-25 and np.signbit(y[0, 2])    # -64 e^-64: tiny, negative
    assert y[0, 3] == P.bf16_round(np.array([1e30]))[0] * 2.0
    assert y[0, 4] == 0.0 and np.signbit(y[0, 4])           # -1e30 / inf = -0
    assert y[0, 5] == 32.0 and y[0, 6] == 256.0


def test_silu_and_mul_against_torch_fp64():
    M, I = 5, 3072
    g = _rows(M, I, seed=7) * 2
    u = _rows(M, I, seed=8)
    y = P.silu_and_mul_ref(np.concatenate([g, u], axis=1))
    t = (F.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    assert np.all(np.abs(y - t) <= 2 * _ulp_bf16(t) + 1e-30)


def test_silu_and_mul_power_of_two_up_scales_exactly():
    g = _rows(2, 512, seed=9)
    ones = np.ones_like(g)
    a = P.silu_and_mul_ref(np.concatenate([g, ones], axis=1))
    for k in (-3, 5):
        y = P.silu_and_mul_ref(np.concatenate([g, ones * 2.0 ** k], axis=1))
        assert np.array_equal(y, a * 2.0 ** k)


def _round_rational_to_bf16(x: Fraction) -> Fraction:
    """Nearest bf16 value to the rational x, ties to the even significand
    (8 significant bits, subnormal spacing 2^-133), in integer arithmetic."""
    if x == 0:
        return Fraction(0)
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()   # 2^e <= a < 2^(e+2)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** max(e - 7, -133)
    n, rem = divmod(a, q)
    if rem * 2 > q or (rem * 2 == q and n % 2 == 1):
        n += 1
    r = n * q
    return r if x > 0 else -r


def test_silu_is_correctly_rounded_for_every_bf16_gate():
    """Every finite bf16 g: bf16(silu(g)) is the bf16 value nearest to the
    exact silu(g), found here from a 50-digit decimal evaluation and an exact
    rational rounding written out in this test (for g >= 100 the answer is g,
    for g <= -100 it is -0)."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    g = (bits << 16).view(np.float32)
    g = g[np.isfinite(g)].astype(np.float64)
    got = P.silu_bf16(g)
    ctx = Context(prec=50, Emin=-10 ** 6, Emax=10 ** 6)
    for gi, yi in zip(g.tolist(), got.tolist()):
        if gi >= 100:
            want = Fraction(gi)
        elif gi <= -100:
            assert yi == 0.0 and math.copysign(1.0, yi) < 0, gi
            continue
        else:
            d = Decimal(gi)
            exact = Fraction(ctx.divide(d, ctx.add(Decimal(1), ctx.exp(-d))))
            want = _round_rational_to_bf16(exact)
        assert Fraction(yi) == want, (gi, yi, float(want))
    # through silu_and_mul_ref with u = 1 as well
    y = P.silu_and_mul_ref(np.concatenate([g[None, :], np.ones((1, g.size))], axis=1))
    assert np.array_equal(y[0], got)


def test_silu_ties_of_tiny_gates_round_towards_plus_infinity():
    """For 0 < |g| < 2^-125 the fp64 value of g / (1 + e^-g) is exactly g / 2.
    silu(g) - g / 2 = g (sigma(g) - 1/2) > 0 for every g != 0, so where g / 2
    lies halfway between two bf16 values the answer is the upper one (for
    g < 0: the one nearer zero); elsewhere it is g / 2 itself."""
    q = 2.0 ** -133
    ks = np.arange(1, 256)                       # |g| = k 2^-133 (subnormal) ...
    mags = np.concatenate([ks * q, (128 + np.arange(128)) * 2.0 ** -133])   # ... and the lowest normal binade
    mags = np.unique(mags[mags < 2.0 ** -125])
    for sign in (1.0, -1.0):
        g = sign * mags
        got = P.silu_bf16(g)
        half = g / 2                              # exact
        n = half / q                              # integer or integer + 1/2
        want = np.where(n == np.floor(n), half, np.ceil(n) * q)   # up at ties (towards +inf)
        assert np.array_equal(got, want), sign
    n = mags / q / 2
    ties = n != np.floor(n)
    assert ties.sum() == 128                                   # odd multiples of 2^-133 on each side
    assert (ties & (np.floor(n) % 2 == 0)).sum() == 64         # of which ties-to-even would go down


# ----------------------------------------------------------------- composition
def test_fused_quant_is_quant_of_the_bf16_output():
    x = _rows(3, 1024, seed=11)
    w = _bf16(np.random.default_rng(11).standard_normal(1024))
    y, _ = P.rms_norm_ref(x, w, 1e-6)
    q, s, _ = P.rms_norm_dynamic_per_token_quant(x, w, 1e-6, "fp8_dynamic")
    q2, s2 = O.quant_per_token(y, "fp8_dynamic")
    assert np.array_equal(q, q2) and np.array_equal(s, s2)
    qb, sb, _ = P.rms_norm_per_block_quant(x, w, 1e-6)
    assert sb.shape == (3, 8)
