"""Plain CPU oracle for the producer-side fused quantizers: RMSNorm or
SiLU-and-multiply followed, in the same kernel, by the dynamic activation
quantization that feeds ``scaled_mm``.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs may import or run this module.  The library under
``quantized_linear_gemm_b200/`` never calls it, links it or shares code with it.

Where the operations come from
------------------------------
The 24-ai.news report "HelionがvLLMに統合：PyTorchネイティブDSLがCUDAカーネルを
代替し、Qwen3モデルのFP8推論を高速化", section "vLLMに統合されたカーネル",
lists, among the nine kernels of the FP8 forward pass,
``rms_norm_dynamic_per_token_quant``, ``silu_and_mul_dynamic_per_token_quant``,
``rms_norm_per_block_quant`` and ``silu_and_mul_per_block_quant``; section
"個別カーネルレベルのパフォーマンス" gives their speed-ups.  The report names the
kernels and nothing more.  The readings below are the plain ones, in the
precision of a bf16 Qwen3 forward pass, and each intermediate rounding is
written out so that the kernels can match the codes bit for bit:

RMSNorm (optionally with the residual added first, the decoder layer's
"add, then normalise"):

* h = bf16(fp32(x + residual))            (or h = x without a residual);
  the new residual is h;
* v = (sum_k h_k^2) / K + eps             in fp64, the sum correctly rounded;
* r = fp32(1 / sqrt(v))                   fp64 sqrt and divide, then rounded;
* y_k = bf16(fp32(bf16(fp32(h_k * r)) * w_k)).

SiLU-and-multiply on the fused gate/up projection output gu = [g | u],
[M, 2I]:

* a_k = bf16(g_k / (1 + exp(-g_k)))       rounded once from the exact value:
  evaluated in fp64, and wherever the fp64 value is too close to a
  midpoint between two bf16 values for its own error to decide the
  rounding, evaluated again with 60 significant decimal digits;
* y_k = bf16(fp32(a_k * u_k))             (the product is exact in fp32).

Then y is quantized with the per-token dynamic rule (FP8 e4m3 or INT8, one
scale per row) or the 1 x 128 group rule (FP8 e4m3, one scale per token and
group), exactly as ``lq_oracle.quant_per_token`` and
``lq_oracle.quant_per_token_group128`` define them.
"""

from __future__ import annotations

import math
from decimal import Context, Decimal
from fractions import Fraction

import numpy as np

from oracle import lq_oracle as O

BF16_MAX = float.fromhex("0x1.fep127")
_BF16_MIN_QUANTUM = 2.0 ** -133   # spacing of bf16 subnormals


def bf16_round(v) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even, with
    one rounding (no detour through fp32).  Returned as float64.  Values at or
    beyond BF16_MAX + half a unit in the last place become +-inf.

    Source: the bf16 rounding of a bf16 decoder layer's intermediates (reading; see the module notes).
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.array(v, copy=True)
    finite = np.isfinite(v) & (v != 0)
    a = np.abs(v[finite])
    e = np.floor(np.log2(a))
    # guard the floor(log2) against rounding at exact powers of two
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    quantum = np.maximum(np.exp2(e - 7), _BF16_MIN_QUANTUM)   # 8 significant bits
    r = np.rint(a / quantum) * quantum                        # a / quantum is exact; rint is half-even
    r = np.where(r > BF16_MAX, np.inf, r)
    out[finite] = np.sign(v[finite]) * r
    return out


def f32(v) -> np.ndarray:
    """Round float64 values to fp32 (nearest, ties to even) and back.

    Source: the fp32 roundings of the same computation (reading; see the module notes).
    """
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def rms_norm_ref(x, weight, eps: float, residual=None):
    """(y, h): the normalised and weighted bf16 row values y [M, K] and the
    (new) residual h [M, K], both as float64 holding bf16 values.  x, weight
    and residual hold bf16 values (float arrays).

    Source: the RMSNorm of ``rms_norm_*_quant``, named in the 24-ai.news report, section
    "vLLMに統合されたカーネル".
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    M, K = x.shape
    if residual is None:
        h = x.copy()
    else:
        h = bf16_round(f32(x + np.asarray(residual, dtype=np.float64)))  # x + res is exact in fp64
    r = np.empty(M, dtype=np.float64)
    eps64 = float(np.float32(eps))
    for m in range(M):
        v = math.fsum(float(t) * float(t) for t in h[m]) / K + eps64
        r[m] = float(np.float32(1.0 / math.sqrt(v)))
    n = bf16_round(f32(h * r[:, None]))        # h * r: exact in fp64 (8 x 24 bits), then fp32, then bf16
    y = bf16_round(f32(n * w[None, :]))        # n * w: exact in fp32 already
    return y, h


def _silu_decimal(g: float, ctx: Context) -> Decimal:
    """silu(g) = g / (1 + e^-g) with 60 significant digits (g exact)."""
    d = Decimal(g)
    return ctx.divide(d, ctx.add(Decimal(1), ctx.exp(ctx.minus(d))))


def _nearest_bf16_to(exact: Decimal, guess: float) -> float:
    """The bf16 value nearest to `exact` among `guess` and its two bf16
    neighbours (ties to the even significand), compared in exact rational
    arithmetic; `guess` is a bf16 value within one unit of the answer."""
    g32 = np.array([guess], dtype=np.float32)
    bits = int(g32.view(np.uint32)[0]) >> 16
    cands = []
    for b in (bits - 1, bits, bits + 1):
        if b < 0:   # below +0: the negative side, -2^-133
            b = 0x8001
        v = float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])
        if math.isfinite(v):
            cands.append((v, b))
    if guess == 0.0:   # +-0: the neighbours on both sides
        cands += [(2.0 ** -133, 1), (-(2.0 ** -133), 0x8001)]
    x = Fraction(exact)   # the 60-digit value, exactly
    best = min(cands, key=lambda c: (abs(x - Fraction(c[0])), c[1] & 1))
    return best[0]


def silu_bf16(g) -> np.ndarray:
    """bf16(silu(g)) for bf16 values g (float64 array), rounded once from the
    exact value of g / (1 + e^-g).

    The fp64 evaluation is within a few units of 2^-52 (relative) of the
    exact value, so its bf16 rounding is the rounding of the exact value
    unless the fp64 value lies within 2^-40 (relative) of a midpoint between
    two bf16 values; those elements are evaluated again with 60 significant
    decimal digits and rounded by exact comparison.  (For |g| < 2^-125 the
    fp64 value is exactly g / 2, a midpoint, while the exact value lies above
    g / 2 since sigma(g) > 1/2 for g > 0 and < 1/2 for g < 0.)

    Source: the SiLU of ``silu_and_mul_*_quant``, named in the 24-ai.news report, section
    "vLLMに統合されたカーネル" (the rounding is a reading: once, from the exact value).
    """
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        s = g / (1.0 + np.exp(-g))
    a = bf16_round(s)
    lo = bf16_round(s * (1.0 - 2.0 ** -40))
    hi = bf16_round(s * (1.0 + 2.0 ** -40))
    unsure = np.flatnonzero((lo != a) | (hi != a))
    if unsure.size:
        ctx = Context(prec=60, Emin=-10 ** 9, Emax=10 ** 9)
        flat = a.reshape(-1)
        gf = g.reshape(-1)
        for i in unsure:
            flat[i] = _nearest_bf16_to(_silu_decimal(float(gf[i]), ctx), float(flat[i]))
    return a


def silu_and_mul_ref(gu):
    """y [M, I] as float64 holding bf16 values, from gu = [g | u] of shape
    [M, 2I] holding bf16 values.

    Source: the SiLU-and-multiply of ``silu_and_mul_*_quant``, named in the 24-ai.news report, section
    "vLLMに統合されたカーネル".
    """
    gu = np.asarray(gu, dtype=np.float64)
    M, two_i = gu.shape
    assert two_i % 2 == 0
    I = two_i // 2
    g, u = gu[:, :I], gu[:, I:]
    a = silu_bf16(g)
    return bf16_round(f32(a * u))


def rms_norm_dynamic_per_token_quant(x, weight, eps: float, fmt: str, residual=None):
    """(codes, scales [M], h): RMSNorm, then per-token quantization.

    Source: 24-ai.news report, section "vLLMに統合されたカーネル".
    """
    y, h = rms_norm_ref(x, weight, eps, residual)
    q, s = O.quant_per_token(y, fmt)
    return q, s, h


def rms_norm_per_block_quant(x, weight, eps: float, residual=None):
    """(codes, scales [M, K/128], h): RMSNorm, then 1 x 128 FP8 quantization.

    Source: 24-ai.news report, section "vLLMに統合されたカーネル".
    """
    y, h = rms_norm_ref(x, weight, eps, residual)
    q, s = O.quant_per_token_group128(y)
    return q, s, h


def silu_and_mul_dynamic_per_token_quant(gu, fmt: str):
    """(codes [M, I], scales [M]).

    Source: 24-ai.news report, section "vLLMに統合されたカーネル".
    """
    return O.quant_per_token(silu_and_mul_ref(gu), fmt)


def silu_and_mul_per_block_quant(gu):
    """(codes [M, I], scales [M, I/128]).

    Source: 24-ai.news report, section "vLLMに統合されたカーネル".
    """
    return O.quant_per_token_group128(silu_and_mul_ref(gu))
