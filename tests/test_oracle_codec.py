"""Pins of the oracle's e4m3 / int8 codecs against the format definition,
hand-worked values and an independent library (torch's float8 cast)."""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O


def _hex(s):
    return int(s, 16)


def test_named_codes_decode(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e4m3_named_codes.json")))
    for item in g["codes"]:
        v = O.e4m3_decode(np.uint8(_hex(item["code"])))
        assert v == item["value"], item
        assert np.signbit(v) == np.signbit(item["value"]), item
    for c in g["nan_codes"]:
        assert np.isnan(O.e4m3_decode(np.uint8(_hex(c))))


def test_named_codes_encode(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e4m3_named_codes.json")))
    for item in g["codes"]:
        c = O.e4m3_encode(np.float32(item["value"]))
        assert int(c) == _hex(item["code"]), item


def test_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (ours == theirs) | (np.isnan(ours) & np.isnan(theirs))
    assert same.all()


def test_decode_int_is_value_times_512():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    ints = O.e4m3_decode_int(codes)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c, i, v in zip(codes, ints, vals):
        assert Fraction(int(i), 512) == Fraction(float(v)), hex(c)
    assert int(np.max(np.abs(ints))) == 229376  # 448 * 2^9 < 2^18


def test_decode_int_rejects_nan():
    with pytest.raises(ValueError):
        O.e4m3_decode_int(np.array([0x7F], dtype=np.uint8))


def test_encode_decode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(O.e4m3_encode(vals), codes)


@pytest.mark.parametrize("v,expect", [
    (1.0625, 0x38),          # midpoint 1 | 1.125 -> even mantissa 0
    (1.1875, 0x3A),          # midpoint 1.125 | 1.25 -> even mantissa 2
    (-1.0625, 0xB8),
    (2.0 ** -10, 0x00),      # midpoint 0 | 2^-9 -> 0
    (3 * 2.0 ** -10, 0x02),  # midpoint 2^-9 | 2*2^-9 -> 2
    (5 * 2.0 ** -10, 0x02),  # midpoint 2*2^-9 | 3*2^-9 -> 2
    (15 * 2.0 ** -10, 0x08), # midpoint 7*2^-9 | 2^-6 -> 2^-6 (mantissa 0 even)
    (232.0, 0x76),           # midpoint 224 | 240 -> 224 (m=6 even)
    (440.0, 0x7E),           # midpoint 432 | 448 -> 448 (m=6 even)
    (1.06251, 0x39),         # just above the midpoint
])
def test_encode_round_half_even(v, expect):
    assert int(O.e4m3_encode(np.float32(v))) == expect


@pytest.mark.parametrize("v,expect", [
    (448.0, 0x7E), (448.5, 0x7E), (463.9, 0x7E), (464.0, 0x7E), (480.0, 0x7E),
    (1e30, 0x7E), (-449.0, 0xFE), (-3.0e38, 0xFE),
])
def test_encode_saturates(v, expect):
    assert int(O.e4m3_encode(np.float32(v))) == expect


def test_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 60,
        rng.standard_normal(20000).astype(np.float32) * 0.01,       # subnormal range
        (rng.integers(-4000, 4000, 20000) * 2.0 ** -12).astype(np.float32),  # many exact ties
    ])
    x = x[np.abs(x) <= 448]
    theirs = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), theirs)


def test_encode_rejects_nonfinite():
    with pytest.raises(ValueError):
        O.e4m3_encode(np.array([np.inf], dtype=np.float32))


@pytest.mark.parametrize("v,expect", [
    (2.5, 2), (-2.5, -2), (3.5, 4), (0.5, 0), (1.5, 2), (-0.5, 0), (126.5, 126),
    (127.49, 127), (127.5, 127), (-127.5, -127), (300.0, 127), (-1e9, -127), (0.49, 0),
])
def test_int8_encode_cases(v, expect):
    assert int(O.int8_encode(np.float32(v))) == expect


def test_int8_encode_matches_python_round():
    # Python's round() on floats is round-half-even, implemented independently of numpy
    rng = np.random.default_rng(2)
    x = (rng.integers(-300, 300, 5000) / 2).astype(np.float32)   # many .5 ties
    x = np.concatenate([x, rng.standard_normal(5000).astype(np.float32) * 80])
    ref = np.array([max(-127, min(127, round(float(v)))) for v in x], dtype=np.int8)
    assert np.array_equal(O.int8_encode(x), ref)
