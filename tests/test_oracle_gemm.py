"""Pins of the oracle's scaled_mm: hand cases, exact-rational brute force with
an independent decoder, the exactness bound, and the invariants that the
blog's variants must satisfy (Split-K and Swap-AB compute the same C;
doubling a scale doubles C; identity weights give back dequant(A))."""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs

FP8 = O.FMT_FP8_DYNAMIC
INT8 = O.FMT_W8A8_INT8
BLK = O.FMT_BLOCK_FP8


def _rows(spec_rows, K, fmt):
    dt = np.int8 if fmt == INT8 else np.uint8
    out = np.zeros((len(spec_rows), K), dtype=dt)
    for i, r in enumerate(spec_rows):
        conv = (lambda v: int(v, 16)) if isinstance(next(iter(r.values())), str) or (
            "set" in r and isinstance(next(iter(r["set"].values())), str)) else int
        if "fill" in r:
            out[i, :] = conv(r["fill"]) if fmt != INT8 else int(r["fill"])
        if "set" in r:
            for k, v in r["set"].items():
                out[i, int(k)] = conv(v) if fmt != INT8 else int(v)
    return out


def test_hand_cases(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gemm_hand_cases.json")))
    for case in g["cases"]:
        fmt, M, N, K = case["fmt"], case["M"], case["N"], case["K"]
        A = _rows(case["A_rows"], K, fmt)
        if "B_rows_all" in case:
            B = _rows([case["B_rows_all"]] * N, K, fmt)
        else:
            B = _rows(case["B_rows"], K, fmt)
        a_s = np.array(case["a_scales"], dtype=np.float32)
        b_s = np.array(case["b_scales"], dtype=np.float32)
        C = O.scaled_mm_ref(fmt, A, a_s, B, b_s)
        if "C_all" in case:
            assert np.all(C == case["C_all"])
        else:
            assert np.array_equal(C, np.array(case["C"], dtype=np.float64)), case
        if "acc" in case:
            assert np.array_equal(O.acc_exact(fmt, A, B), np.array(case["acc"]))


def _torch_decode_fraction(fmt, codes):
    """Exact operand values through an independent decoder (torch's fp8 / int8 views)."""
    if fmt == INT8:
        return [[Fraction(int(v)) for v in row] for row in codes]
    vals = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return [[Fraction(float(v)) for v in row] for row in vals]


def _random_codes(fmt, shape, rng):
    if fmt == INT8:
        return rng.integers(-127, 128, shape).astype(np.int8)
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x7E   # no NaN codes in operands
    return c


@pytest.mark.parametrize("fmt", [FP8, INT8, BLK])
def test_bruteforce_fraction_2x3x256(fmt):
    rng = np.random.default_rng({FP8: 10, INT8: 11, BLK: 12}[fmt])
    M, N, K = 2, 3, 256
    A = _random_codes(fmt, (M, K), rng)
    B = _random_codes(fmt, (N, K), rng)
    if fmt == BLK:
        # N = 3 is not a multiple of 128: a per-(n-block, k-block) scale still
        # has one n-block; the oracle indexes it as n // 128
        a_s = (rng.random((M, 2)) + 0.1).astype(np.float32)
        b_s = (rng.random((1, 2)) + 0.1).astype(np.float32)
    else:
        a_s = (rng.random(M) + 0.1).astype(np.float32)
        b_s = (rng.random(N) + 0.1).astype(np.float32)
    Af = _torch_decode_fraction(fmt, A)
    Bf = _torch_decode_fraction(fmt, B)
    C = O.scaled_mm_ref(fmt, A, a_s, B, b_s)
    for m in range(M):
        for n in range(N):
            if fmt == BLK:
                exact = sum(
                    sum(Af[m][k] * Bf[n][k] for k in range(kb * 128, kb * 128 + 128))
                    * Fraction(float(a_s[m, kb])) * Fraction(float(b_s[0, kb]))
                    for kb in range(2))
            else:
                exact = sum(Af[m][k] * Bf[n][k] for k in range(K)) * Fraction(float(a_s[m])) * Fraction(float(b_s[n]))
            # fp64 scaling of an exact integer: a few ulps of relative error at most
            assert abs(Fraction(float(C[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


def test_accumulator_exact_at_extremes():
    """K = 25600 of the largest codes: the int64 sum equals the Python integer."""
    K = 25600
    A = np.full((1, K), 0x7E, dtype=np.uint8)
    B = np.full((2, K), 0x7E, dtype=np.uint8)
    B[1, :] = 0xFE
    acc = O.acc_exact(FP8, A, B)
    assert int(acc[0, 0]) == K * 229376 * 229376
    assert int(acc[0, 1]) == -K * 229376 * 229376
    assert abs(int(acc[0, 0])) < 2 ** 51
    Ai = np.full((1, K), -127, dtype=np.int8)
    Bi = np.full((1, K), -127, dtype=np.int8)
    assert int(O.acc_exact(INT8, Ai, Bi)[0, 0]) == K * 127 * 127 < 2 ** 31


@pytest.mark.parametrize("fmt", [FP8, INT8])
@pytest.mark.parametrize("K", [128, 1024, 1040])   # 1040: a ragged last K tile
def test_split_k_equals_standard(fmt, K):
    rng = np.random.default_rng(K)
    A = _random_codes(fmt, (5, K), rng)
    B = _random_codes(fmt, (7, K), rng)
    ref = O.acc_exact(fmt, A, B)
    for S in (1, 2, 4, 8, 16, 32, 64, 128, 256):
        assert np.array_equal(O.acc_split_k(fmt, A, B, S), ref), S


def test_split_ranges_cover_and_allow_empty():
    for T in (1, 3, 40, 96, 200):
        for S in (1, 2, 4, 64, 256):
            r = O.split_ranges(T, S)
            assert r[0][0] == 0 and r[-1][1] == T
            assert all(r[i][1] == r[i + 1][0] for i in range(S - 1))
            assert sum(hi - lo for lo, hi in r) == T
            if S > T:
                assert any(hi == lo for lo, hi in r)


@pytest.mark.parametrize("fmt", [FP8, INT8])
def test_swap_ab_equals_standard(fmt):
    rng = np.random.default_rng(20)
    A = _random_codes(fmt, (3, 96), rng)
    B = _random_codes(fmt, (9, 96), rng)
    assert np.array_equal(O.acc_swap_ab(fmt, A, B), O.acc_exact(fmt, A, B))


@pytest.mark.parametrize("fmt", [FP8, INT8])
def test_transposed_product(fmt):
    """Exchanging the operands' roles gives C^T (scales exchanged with them)."""
    rng = np.random.default_rng(21)
    A = _random_codes(fmt, (4, 128), rng)
    B = _random_codes(fmt, (6, 128), rng)
    a_s = (rng.random(4) + 0.5).astype(np.float32)
    b_s = (rng.random(6) + 0.5).astype(np.float32)
    C = O.scaled_mm_ref(fmt, A, a_s, B, b_s)
    Ct = O.scaled_mm_ref(fmt, B, b_s, A, a_s)
    assert np.allclose(C, Ct.T, rtol=1e-15, atol=0)


@pytest.mark.parametrize("fmt", [FP8, INT8, BLK])
def test_scale_linearity(fmt):
    rng = np.random.default_rng(22)
    K = 256
    A = _random_codes(fmt, (4, K), rng)
    B = _random_codes(fmt, (128, K), rng)
    if fmt == BLK:
        a_s = (rng.random((4, 2)) + 0.5).astype(np.float32)
        b_s = (rng.random((1, 2)) + 0.5).astype(np.float32)
    else:
        a_s = (rng.random(4) + 0.5).astype(np.float32)
        b_s = (rng.random(128) + 0.5).astype(np.float32)
    C = O.scaled_mm_ref(fmt, A, a_s, B, b_s)
    a2 = a_s.copy()
    a2[2] *= 2
    C2 = O.scaled_mm_ref(fmt, A, a2, B, b_s)
    assert np.array_equal(C2[2], 2 * C[2])
    keep = [0, 1, 3]
    assert np.array_equal(C2[keep], C[keep])


def test_identity_weights_give_dequantized_activations():
    x = inputs.activations(4, 256, seed=23).float().numpy()
    q, s = O.quant_per_token(x, FP8)
    eye = np.where(np.eye(256, dtype=bool), 0x38, 0x00).astype(np.uint8)   # B = I (1.0 on the diagonal)
    C = O.scaled_mm_ref(FP8, q, s, eye, np.ones(256, dtype=np.float32))
    assert np.array_equal(C, O.e4m3_decode(q) * s[:, None].astype(np.float64))


def test_blockwise_with_uniform_scales_equals_per_token_form():
    """With every block scale of a row equal, Block_FP8 reduces to FP8_Dynamic."""
    rng = np.random.default_rng(24)
    A = _random_codes(FP8, (3, 384), rng)
    B = _random_codes(FP8, (256, 384), rng)
    a_row = (rng.random(3) + 0.5).astype(np.float32)
    b_blk = (rng.random(2) + 0.5).astype(np.float32)
    Cb = O.blockwise_ref(A, np.repeat(a_row[:, None], 3, axis=1), B, np.repeat(b_blk[:, None], 3, axis=1))
    Cp = O.scaled_mm_ref(FP8, A, a_row, B, np.repeat(b_blk, 128))
    # the two differ only by fp64 rounding of the per-block scaled partial sums
    assert np.allclose(Cb, Cp, rtol=0, atol=1e-12 * float(np.max(np.abs(Cp))))


def test_tolerance_rejects_planted_mistakes():
    """The acceptance bound is tight enough to catch the usual slips: a
    transposed operand, a dropped K tile, a sign error, a missing scale."""
    x = inputs.activations(8, 512, seed=25).float().numpy()
    w = inputs.weights(256, 512, seed=26).float().numpy()
    qa, sa = O.quant_per_token(x, FP8)
    qb, sb = O.quant_per_channel(w, FP8)
    C = O.scaled_mm_ref(FP8, qa, sa, qb, sb)
    bf = torch.from_numpy(C).to(torch.bfloat16).to(torch.float64).numpy()
    assert O.within_tolerance(bf, C)[0]
    qb_drop = qb.copy()
    qb_drop[:, 128:256] = 0                                               # one K tile dropped
    bad_drop = O.scaled_mm_ref(FP8, qa, sa, qb_drop, sb)
    bad_scale = O.scaled_mm_ref(FP8, qa, np.ones_like(sa), qb, sb)
    for bad in (-C, bad_drop, bad_scale):
        assert not O.within_tolerance(bad, C)[0]
    # a transposed / reversed K axis of one operand
    assert not O.within_tolerance(O.scaled_mm_ref(FP8, qa, sa, qb[:, ::-1], sb), C)[0]


def test_bf16_rounding_within_tolerance_at_qwen_shape_sample():
    """The correctly rounded bf16 of C_ref always passes: 2^-8 < 2^-7."""
    x = inputs.activations(4, 4096, seed=27).float().numpy()
    w = inputs.weights(64, 4096, seed=28).float().numpy()
    qa, sa = O.quant_per_token(x, INT8)
    qb, sb = O.quant_per_channel(w, INT8)
    C = O.scaled_mm_ref(INT8, qa, sa, qb, sb)
    bf = torch.from_numpy(C).to(torch.bfloat16).to(torch.float64).numpy()
    ok, worst = O.within_tolerance(bf, C)
    assert ok and worst <= 0.5 + 1e-9
