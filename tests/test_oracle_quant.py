"""Pins of the oracle's quantizers: hand-worked rows, the scale floor, the
amax element, and the dequantization error bound that the rounding implies."""

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
