"""Pins of the oracle's quantizers: hand-worked rows, the scale floor, the
amax element, the dequantization error bound that the rounding implies, and
rows where only the correctly rounded quotient x / s (not x * (1 / s)) gives
the right code, checked in exact rational arithmetic."""

import json
import os

import numpy as np
import pytest

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs


def _codes(fmt, raw):
    if fmt == O.FMT_W8A8_INT8:
        return np.array(raw, dtype=np.int8)
    return np.array([int(c, 16) for c in raw], dtype=np.uint8)


def test_hand_rows(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "quant_rows.json")))
    for row in g["rows"]:
        x = np.array([row["x"]], dtype=np.float32)
        q, s = O.quant_per_token(x, row["fmt"])
        assert s.shape == (1,)
        assert float(s[0]) == np.float32(row["scale"]), row
        assert np.array_equal(q[0], _codes(row["fmt"], row["codes"])), row


@pytest.mark.parametrize("fmt", [O.FMT_FP8_DYNAMIC, O.FMT_W8A8_INT8])
def test_amax_element_maps_to_qmax(fmt):
    x = inputs.activations(16, 512, seed=3).float().numpy()
    q, s = O.quant_per_token(x, fmt)
    idx = np.argmax(np.abs(x), axis=1)
    top = q[np.arange(16), idx]
    if fmt == O.FMT_W8A8_INT8:
        assert np.all(np.abs(top.astype(np.int64)) == 127)
    else:
        assert np.all((top & 0x7F) == 0x7E)


@pytest.mark.parametrize("fmt", [O.FMT_FP8_DYNAMIC, O.FMT_W8A8_INT8, O.FMT_BLOCK_FP8])
def test_dequant_error_bound(fmt):
    """|dequant(q) - x| is at most half a quantum of the code grid.

    e4m3: relative 2^-4 for normal codes, absolute 2^-10 * s below 2^-6 * s;
    int8: absolute s/2.  A wrong scale, a reciprocal-vs-division slip of more
    than an ulp, or a dropped sign all break this bound."""
    x = inputs.activations(8, 1024, seed=4).float().numpy()
    if fmt == O.FMT_BLOCK_FP8:
        q, s = O.quant_per_token_group128(x)
        s_full = np.repeat(s, 128, axis=1)
    else:
        q, s = O.quant_per_token(x, fmt)
        s_full = np.repeat(s[:, None], x.shape[1], axis=1)
    if fmt == O.FMT_W8A8_INT8:
        deq = q.astype(np.float64) * s_full
        bound = 0.5 * s_full * (1 + 1e-6) + 1e-30
    else:
        deq = O.e4m3_decode(q) * s_full
        mag = np.abs(x.astype(np.float64)) / s_full
        bound = np.where(mag >= 2.0 ** -6, 2.0 ** -4 * np.abs(x), 2.0 ** -10 * s_full) * (1 + 1e-6) + 1e-30
    assert np.all(np.abs(deq - x) <= bound)


def test_zero_row_uses_scale_floor():
    x = np.zeros((2, 256), dtype=np.float32)
    for fmt in (O.FMT_FP8_DYNAMIC, O.FMT_W8A8_INT8):
        q, s = O.quant_per_token(x, fmt)
        assert np.all(s == np.float32(2.0 ** -126))
        assert np.all(q.view(np.uint8) == 0)


def test_tiny_row_scale_floor_is_applied():
    # amax / 448 would be subnormal in fp32: the scale is clamped to 2^-126
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 5] = np.float32(1e-37)
    q, s = O.quant_per_token(x, O.FMT_FP8_DYNAMIC)
    assert s[0] == np.float32(2.0 ** -126)
    assert O.e4m3_decode(q[0, 5]) * float(s[0]) == pytest.approx(1e-37, rel=2 ** -3)


def test_group128_is_per_token_on_each_group():
    x = inputs.activations(3, 384, seed=5).float().numpy()
    q, s = O.quant_per_token_group128(x)
    assert s.shape == (3, 3)
    for g in range(3):
        qg, sg = O.quant_per_token(x[:, g * 128:(g + 1) * 128], O.FMT_BLOCK_FP8)
        assert np.array_equal(q[:, g * 128:(g + 1) * 128], qg)
        assert np.array_equal(s[:, g], sg)


def test_group128_hand_case():
    x = np.zeros((1, 256), dtype=np.float32)
    x[0, 0] = 448.0        # group 0: s = 1
    x[0, 1] = -1.0
    x[0, 128] = 44.8       # group 1: s = fp32(44.8/448) = fp32(0.1)
    q, s = O.quant_per_token_group128(x)
    assert s[0, 0] == 1.0
    assert s[0, 1] == np.float32(np.float32(44.8) / np.float32(448.0))
    assert q[0, 0] == 0x7E and q[0, 1] == 0xB8 and q[0, 128] == 0x7E


def test_weight_block128_hand_case():
    w = np.zeros((256, 256), dtype=np.float32)
    w[0, 0] = 448.0          # block (0,0): s = 1
    w[130, 3] = -896.0       # block (1,0): s = 2
    w[7, 200] = 4.48         # block (0,1): s = fp32(0.01)
    q, s = O.quant_weight_block128(w)
    assert s.shape == (2, 2)
    assert s[0, 0] == 1.0 and s[1, 0] == 2.0
    assert s[0, 1] == np.float32(np.float32(4.48) / np.float32(448.0))
    assert s[1, 1] == np.float32(2.0 ** -126)
    assert q[0, 0] == 0x7E and q[130, 3] == 0xFE and q[7, 200] == 0x7E
    assert np.count_nonzero(q) == 3


def test_weight_block128_amax_over_whole_block():
    w = inputs.weights(256, 384, seed=6).float().numpy()
    q, s = O.quant_weight_block128(w)
    for nb in range(2):
        for kb in range(3):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert s[nb, kb] == np.float32(np.float32(np.max(np.abs(blk))) / np.float32(448.0))
            assert np.max(q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128] & 0x7F) == 0x7E


def test_per_channel_weight_is_per_row():
    w = inputs.weights(5, 256, seed=7).float().numpy()
    q, s = O.quant_per_channel(w, O.FMT_W8A8_INT8)
    assert s.shape == (5,)
    for n in range(5):
        assert s[n] == np.float32(np.float32(np.max(np.abs(w[n]))) / np.float32(127.0))


# ---------------------------------------------------------------------------
# The code is enc(RN32(x / s)), the correctly rounded quotient, not
# x * RN32(1 / s).  The two differ in the last fp32 bit for some x, and the
# code differs when that bit straddles a rounding boundary of the code grid.
# The hand rows above use power-of-two scales, where both agree; these rows
# are found by a search over bf16 values and checked in exact rational
# arithmetic (an fp32 rounding and both encoders written out here, apart from
# the oracle's).

from fractions import Fraction  # noqa: E402

import torch  # noqa: E402


def _rn32(f: Fraction) -> Fraction:
    """Nearest fp32 value of a rational (ties to even; normal and subnormal range)."""
    if f == 0:
        return Fraction(0)
    sign, a = (-1, -f) if f < 0 else (1, f)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    n, rem = divmod(a / quantum, 1)
    n = int(n)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2):
        n += 1
    return sign * n * quantum


def _e4m3_exact(y: Fraction) -> Fraction:
    """Value of the e4m3 code of y: round to nearest even on the 3-bit
    significand (subnormal quantum 2^-9), saturating at +-448."""
    if y == 0:
        return Fraction(0)
    sign, a = (-1, -y) if y < 0 else (1, y)
    if a >= 448:
        return sign * Fraction(448)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    quantum = Fraction(2) ** (max(e, -6) - 3)
    n, rem = divmod(a / quantum, 1)
    n = int(n)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2):
        n += 1
    return sign * min(Fraction(448), n * quantum)


def _int8_exact(y: Fraction) -> int:
    return max(-127, min(127, round(y)))   # Fraction rounds half to even


def _bf16_grid():
    bits = np.arange(0x0080, 0x7F80, dtype=np.uint32)   # every positive normal bf16
    return (bits << 16).view(np.float32)


def _straddling_rows(fmt, limit=16):
    """(amax, x) bf16 pairs, |x| <= amax, whose codes under x / s and under
    x * (1 / s) differ (found with numpy fp32 arithmetic and torch's cast)."""
    Q = np.float32(448.0 if fmt == O.FMT_FP8_DYNAMIC else 127.0)
    vals = _bf16_grid()
    rows = []
    for amax in vals[(vals >= 1) & (vals < 4)]:
        s = np.float32(amax) / Q
        xs = vals[(vals <= amax) & (vals >= amax / 256)]
        yd, yr = xs / s, xs * (np.float32(1) / s)
        if fmt == O.FMT_FP8_DYNAMIC:
            cd = torch.from_numpy(yd).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            cr = torch.from_numpy(yr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        else:
            cd, cr = np.rint(yd), np.rint(yr)
        rows += [(float(amax), float(xs[i])) for i in np.nonzero(cd != cr)[0][:1]]
        if len(rows) >= limit:
            break
    return rows


@pytest.mark.parametrize("fmt", [O.FMT_FP8_DYNAMIC, O.FMT_W8A8_INT8])
def test_codes_use_the_correctly_rounded_quotient(fmt):
    Q = 448 if fmt == O.FMT_FP8_DYNAMIC else 127
    rows = _straddling_rows(fmt)
    assert len(rows) >= 8   # the check below can tell the two quotients apart
    for amax, x in rows:
        q, s = O.quant_per_token(np.array([[amax, x]], dtype=np.float32), fmt)
        s_exact = _rn32(Fraction(amax) / Q)
        assert Fraction(float(s[0])) == s_exact
        y_div = _rn32(Fraction(x) / s_exact)
        y_rcp = _rn32(Fraction(x) * _rn32(1 / s_exact))
        if fmt == O.FMT_FP8_DYNAMIC:
            got = Fraction(float(torch.from_numpy(q[0].copy()).view(torch.float8_e4m3fn)[1].to(torch.float64)))
            want, wrong = _e4m3_exact(y_div), _e4m3_exact(y_rcp)
        else:
            got, want, wrong = int(q[0, 1]), _int8_exact(y_div), _int8_exact(y_rcp)
        assert want != wrong, (amax, x)
        assert got == want, (amax, x, got, want)


def test_exact_helpers_on_known_values():
    """The rational helpers of the check above, on values fixed by hand."""
    assert _rn32(Fraction(1, 3)) == Fraction(11184811, 2 ** 25)     # 0x3EAAAAAB
    assert _rn32(Fraction(2 ** 24 + 1)) == 2 ** 24                   # tie to even
    assert _rn32(Fraction(2 ** 24 + 3)) == 2 ** 24 + 4               # tie to even, upwards
    assert _rn32(Fraction(1, 2 ** 149)) == Fraction(1, 2 ** 149)     # smallest subnormal
    assert _e4m3_exact(Fraction(17, 16)) == 1                        # 1.0625: tie, to even (1.0)
    assert _e4m3_exact(Fraction(19, 16)) == Fraction(5, 4)           # 1.1875: tie, to even (1.25)
    assert _e4m3_exact(Fraction(460)) == 448 and _e4m3_exact(Fraction(-1000)) == -448
    assert _e4m3_exact(Fraction(3, 2 ** 10)) == Fraction(2, 2 ** 9)  # subnormal tie 1.5 quanta -> 2
    assert _int8_exact(Fraction(5, 2)) == 2 and _int8_exact(Fraction(-7, 2)) == -4
