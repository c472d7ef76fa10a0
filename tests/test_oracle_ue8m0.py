"""Pins of the UE8M0 (power-of-two scale) Block_FP8 oracle against things
other than itself: the e8m0 closed form, the smallest-power-of-two rule
checked by exact rational search, the no-saturation / minimality property
of the codes, and an exact rational brute-force product.  CPU only."""

from fractions import Fraction

import numpy as np
import torch

from oracle import lq_oracle as O
from oracle import ue8m0_oracle as U
from quantized_linear_gemm_b200 import inputs


def test_e8m0_named_values():
    assert U.e8m0_decode([127])[0] == 1.0
    assert U.e8m0_decode([128])[0] == 2.0
    assert U.e8m0_decode([126])[0] == 0.5
    assert U.e8m0_decode([0])[0] == 2.0 ** -127
    assert U.e8m0_decode([254])[0] == 2.0 ** 127
    assert np.isnan(U.e8m0_decode([255])[0])


def _smallest_e(amax: float) -> int:
    """By exact rational search: the smallest e with amax <= 448 * 2^e."""
    a = Fraction(amax)
    if a == 0:
        return -127
    e = -200
    while a > 448 * Fraction(2) ** e:
        e += 1
    return max(-127, min(127, e))


def test_exponent_rule_by_rational_search():
    g = np.random.default_rng(1)
    vals = (np.abs(g.standard_normal(3000)) * np.exp2(g.integers(-140, 127, 3000))).astype(np.float32)
    vals = np.concatenate([vals, np.float32([0.0, 448.0, 448.0 * 2 ** -20, 1e-45, 3e38])])
    for k in (-30, -1, 0, 5, 40):                          # exactly 448 * 2^k and its neighbours
        t = np.float32(448.0 * 2.0 ** k)
        vals = np.concatenate([vals, [t, np.nextafter(t, np.float32(np.inf)), np.nextafter(t, np.float32(0))]])
    e = U.ue8m0_exponent(vals.astype(np.float64))
    for v, ev in zip(vals, e):
        assert ev == _smallest_e(float(v)), v


def test_codes_never_saturate_and_the_scale_is_minimal():
    x = inputs.activations(16, 1024, seed=2).float().numpy()
    q, b = U.quant_per_token_group128_ue8m0(x)
    vals = O.e4m3_decode(q).reshape(16, 8, 128)
    assert np.all(np.abs(vals) <= 448)
    s = U.e8m0_decode(b)
    g = x.reshape(16, 8, 128).astype(np.float64)
    amax = np.abs(g).max(-1)
    assert np.all(amax / s <= 448)            # no element beyond the largest code
    assert np.all(amax / (s / 2) > 448)       # half the scale would saturate: s is the smallest
    # dequantization error within half an e4m3 step of each value's binade
    deq = vals * s[..., None]
    step = np.maximum(np.exp2(np.floor(np.log2(np.maximum(np.abs(g / s[..., None]), 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(deq - g) <= step / 2 * s[..., None] + 1e-300)


def test_zero_group_and_exact_power_of_two_group():
    x = np.zeros((2, 256), dtype=np.float32)
    x[1, :128] = 448.0 * 2.0 ** -3          # amax exactly 448 * 2^-3: e = -3, every code is 448
    q, b = U.quant_per_token_group128_ue8m0(x)
    assert b[0, 0] == 0 and b[0, 1] == 0 and b[1, 1] == 0 and np.all(q[0] == 0)
    assert b[1, 0] == 127 - 3 and np.all(q[1, :128] == 0x7E)


def test_weight_blocks_use_the_whole_block():
    w = inputs.weights(256, 384, seed=3).float().numpy()
    q, b = U.quant_weight_block128_ue8m0(w)
    assert b.shape == (2, 3)
    blocks = w.reshape(2, 128, 3, 128)
    for nb in range(2):
        for kb in range(3):
            assert b[nb, kb] == U.ue8m0_exponent(np.abs(blocks[nb, :, kb, :]).max()) + 127


def test_blockwise_product_by_exact_rational_brute_force():
    M, N, K = 2, 128, 256
    x = inputs.activations(M, K, seed=4).float().numpy()
    w = inputs.weights(N, K, seed=5).float().numpy()
    qa, ba = U.quant_per_token_group128_ue8m0(x)
    qb, bb = U.quant_weight_block128_ue8m0(w)
    C = U.blockwise_ue8m0_ref(qa, ba, qb, bb)
    dec = lambda c: [Fraction(float(v)) for v in torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).to(torch.float64)]
    for m in range(M):
        for n in (0, 17, 127):
            total = Fraction(0)
            for kb in range(K // 128):
                av = dec(qa[m, kb * 128:(kb + 1) * 128])
                bv = dec(qb[n, kb * 128:(kb + 1) * 128])
                sa = Fraction(2) ** (int(ba[m, kb]) - 127)
                sb = Fraction(2) ** (int(bb[0, kb]) - 127)
                total += sum(p * r for p, r in zip(av, bv)) * sa * sb
            assert C[m, n] == float(total)
