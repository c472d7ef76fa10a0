"""Pins of the grouped (MoE) quantized GEMM oracle against things other
than itself: exact rational brute force with torch's own e4m3 decoder, the
single-expert case (the pinned dense oracle), block structure invariants,
and offset validation.  CPU only."""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from oracle import moe_oracle as MO
from quantized_linear_gemm_b200 import inputs


def _problem(fmt, counts, N, K, seed):
    g = np.random.default_rng(seed)
    T, E = int(sum(counts)), len(counts)
    x = g.standard_normal((T, K)).astype(np.float32)
    w = (0.02 * g.standard_normal((E, N, K))).astype(np.float32)
    a, sa = O.quant_per_token(x, fmt) if T else (np.zeros((0, K), np.uint8), np.zeros(0, np.float32))
    b = np.empty((E, N, K), dtype=np.int8 if fmt == "w8a8_int8" else np.uint8)
    sb = np.empty((E, N), dtype=np.float32)
    for e in range(E):
        b[e], sb[e] = O.quant_per_channel(w[e], fmt)
    off = np.concatenate([[0], np.cumsum(counts)])
    return a, sa, b, sb, off


def _dec(codes, fmt):
    if fmt == "w8a8_int8":
        return [int(v) for v in np.asarray(codes, dtype=np.int8).ravel()]
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8).ravel().copy()).view(torch.float8_e4m3fn)
    return [Fraction(float(v)) for v in t.to(torch.float64)]


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
def test_grouped_matches_exact_rational_brute_force(fmt):
    counts = [2, 0, 3, 1]                       # an expert with no token
    N, K = 3, 32
    a, sa, b, sb, off = _problem(fmt, counts, N, K, seed=1)
    C = MO.grouped_scaled_mm_ref(fmt, a, sa, b, sb, off)
    for e in range(len(counts)):
        for t in range(off[e], off[e + 1]):
            av = _dec(a[t], fmt)
            for n in range(N):
                bv = _dec(b[e, n], fmt)
                exact = sum(x * y for x, y in zip(av, bv)) * Fraction(float(sa[t])) * Fraction(float(sb[e, n]))
                assert C[t, n] == float(exact), (e, t, n)


def test_single_expert_is_the_dense_product():
    a, sa, b, sb, off = _problem("fp8_dynamic", [7], 16, 256, seed=2)
    C = MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b, sb, off)
    assert np.array_equal(C, O.scaled_mm_ref("fp8_dynamic", a, sa, b[0], sb[0]))


def test_rows_depend_only_on_their_expert():
    counts = [3, 2, 4]
    a, sa, b, sb, off = _problem("fp8_dynamic", counts, 8, 128, seed=3)
    C = MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b, sb, off)
    b2 = b.copy()
    b2[1] = np.roll(b2[1], 1, axis=0)
    C2 = MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b2, sb, off)
    assert np.array_equal(C[:3], C2[:3]) and np.array_equal(C[5:], C2[5:])
    assert not np.array_equal(C[3:5], C2[3:5])


def test_permuting_experts_permutes_row_blocks():
    counts = [3, 1, 4]
    a, sa, b, sb, off = _problem("w8a8_int8", counts, 8, 128, seed=4)
    C = MO.grouped_scaled_mm_ref("w8a8_int8", a, sa, b, sb, off)
    perm = [2, 0, 1]
    blocks = [np.arange(off[e], off[e + 1]) for e in range(3)]
    rows = np.concatenate([blocks[e] for e in perm])
    off_p = np.concatenate([[0], np.cumsum([counts[e] for e in perm])])
    Cp = MO.grouped_scaled_mm_ref("w8a8_int8", a[rows], sa[rows], b[perm], sb[perm], off_p)
    assert np.array_equal(Cp, C[rows])


@pytest.mark.parametrize("off", [[1, 3, 5], [0, 4, 3], [0, 2, 6], [0, 5]])
def test_bad_offsets_are_rejected(off):
    a, sa, b, sb, _ = _problem("fp8_dynamic", [2, 3], 4, 32, seed=5)
    with pytest.raises(ValueError):
        MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b, sb, off)


def test_expert_counts_generator():
    c = inputs.expert_counts(64, 128, 8, seed=6)
    assert c.sum() == 64 * 8 and c.shape == (128,) and c.min() >= 0
    assert np.array_equal(c, inputs.expert_counts(64, 128, 8, seed=6))
