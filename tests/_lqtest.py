"""Shared helpers of the GPU parity tests: seeded problems quantized by the
oracle on the CPU, the same codes copied to the GPU, and the comparison
against the oracle's fp64 reference."""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from oracle import lq_oracle as O
from oracle import ue8m0_oracle as U
from quantized_linear_gemm_b200 import inputs, lq

FMT_NAME = {lq.FP8_DYNAMIC: O.FMT_FP8_DYNAMIC, lq.W8A8_INT8: O.FMT_W8A8_INT8, lq.BLOCK_FP8: O.FMT_BLOCK_FP8}


@dataclass
class Problem:
    fmt: int
    M: int
    N: int
    K: int
    qa: np.ndarray
    sa: np.ndarray
    qb: np.ndarray
    sb: np.ndarray

    def device(self, dev="cuda"):
        """(A, a_scales, B, b_scales) on the GPU: uint8 e4m3 codes or int8 codes, fp32 scales."""
        A = torch.from_numpy(np.ascontiguousarray(self.qa)).to(dev)
        B = torch.from_numpy(np.ascontiguousarray(self.qb)).to(dev)
        sdt = np.uint8 if self.fmt == lq.BLOCK_FP8_UE8M0 else np.float32   # UE8M0 scales are bytes
        sa = torch.from_numpy(np.ascontiguousarray(self.sa, dtype=sdt)).to(dev)
        sb = torch.from_numpy(np.ascontiguousarray(self.sb, dtype=sdt)).to(dev)
        return A, sa, B, sb

    def reference(self, rows=None, cols=None):
        qa, sa, qb, sb = self.qa, self.sa, self.qb, self.sb
        if self.fmt == lq.BLOCK_FP8_UE8M0:   # the decoded power-of-two scales, then as Block_FP8
            sa, sb = U.e8m0_decode(sa), U.e8m0_decode(sb)
        if rows is not None:
            qa, sa = qa[rows], sa[rows]
        block = self.fmt in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0)
        if cols is not None:
            qb = qb[cols]
            if not block:
                sb = sb[cols]
        if block and cols is not None:
            # keep the n-block scale of each sampled column: expand to per-column blocks
            return _block_ref_cols(qa, sa, qb, sb, np.asarray(cols))
        if block:
            return O.blockwise_ref(qa, sa, qb, sb)
        return O.scaled_mm_ref(FMT_NAME[self.fmt], qa, sa, qb, sb)


def _block_ref_cols(qa, sa, qb_cols, sb, cols):
    """Block_FP8 reference for sampled weight rows: each sampled row n keeps its block scale row n // 128."""
    out = np.zeros((qa.shape[0], len(cols)), dtype=np.float64)
    for j, n in enumerate(cols):
        nb = int(n) // 128
        out[:, j] = O.blockwise_ref(qa, sa, qb_cols[j:j + 1], sb[nb:nb + 1])[:, 0]
    return out


def make_problem(fmt: int, M: int, N: int, K: int, seed: int, outliers: bool = True) -> Problem:
    x = inputs.activations(M, K, seed=inputs.stable_seed("A", fmt, M, N, K, seed), outliers=outliers).float().numpy()
    w = inputs.weights(N, K, seed=inputs.stable_seed("B", fmt, M, N, K, seed)).float().numpy()
    if fmt == lq.BLOCK_FP8_UE8M0:
        qa, sa = U.quant_per_token_group128_ue8m0(x)
        qb, sb = U.quant_weight_block128_ue8m0(w)
        return Problem(fmt, M, N, K, qa, sa, qb, sb)
    name = FMT_NAME[fmt]
    if fmt == lq.BLOCK_FP8:
        qa, sa = O.quant_per_token_group128(x)
        qb, sb = O.quant_weight_block128(w)
    else:
        qa, sa = O.quant_per_token(x, name)
        qb, sb = O.quant_per_channel(w, name)
    return Problem(fmt, M, N, K, qa, sa, qb, sb)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(C_gpu: torch.Tensor, C_ref: np.ndarray, what: str = "", rms_of=None):
    C = bf16_to_f64(C_gpu) if isinstance(C_gpu, torch.Tensor) else C_gpu
    assert C.shape == C_ref.shape, (C.shape, C_ref.shape)
    assert np.all(np.isfinite(C)), f"{what}: non-finite output"
    ok, worst = O.within_tolerance(C, C_ref, rms_of=rms_of)
    if not ok:
        err = np.abs(C - C_ref)
        i = np.unravel_index(np.argmax(err), err.shape)
        raise AssertionError(f"{what}: outside tolerance, worst ratio {worst:.3g} at {i}: gpu {C[i]!r} ref {C_ref[i]!r}")
    return worst


def wide_range_rows(K: int, seed: int) -> torch.Tensor:
    """bf16 rows that exercise both ways the kernels divide by the scale: the
    FMA-corrected reciprocal (amax >= 2^-80) and the plain division (smaller
    amax), around the 2^-80 boundary, with elements down to bf16 subnormals
    and up to 2^120, and rows whose every scale is extreme."""
    g = np.random.default_rng(seed)
    rows = []
    def row(lo, hi, amax=None):
        e = g.uniform(lo, hi, K)
        v = np.where(g.random(K) < 0.5, -1.0, 1.0)
        r = v * (1.0 + g.random(K)) * np.exp2(e)
        if amax is not None:
            r[g.integers(K)] = amax
        return r
    rows.append(row(-140, -81, amax=2.0 ** -80))                 # amax exactly 2^-80: fast path
    rows.append(row(-140, -82, amax=-(2.0 ** -80) * (1 - 2 ** -8)))   # just below: division
    rows.append(row(-133, -100))                                # all tiny, subnormals included
    rows.append(row(-130, 100))                                 # 230 binades in one row
    rows.append(row(60, 120, amax=3.0e38))                      # scale near the top of fp32
    rows.append(row(-20, 5))
    x = torch.from_numpy(np.stack(rows)).to(torch.bfloat16)
    return x
