"""Full-size parity at the Qwen3 linear shapes, in the launch configuration
the benchmark times (variant = the dispatch table's choice), checked on
sampled outputs that the oracle computes one by one.

Weights are quantized by the oracle once per shape (module-scoped cache) and
the same codes are given to the GPU."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from oracle import ue8m0_oracle as U

from _lqtest import FMT_NAME, assert_close

pytestmark = pytest.mark.gpu

_cache = {}


def _weights(fmt, N, K):
    key = (fmt, N, K)
    if key not in _cache:
        w = inputs.weights(N, K, seed=inputs.stable_seed("full-W", fmt, N, K)).float().numpy()
        if fmt == lq.BLOCK_FP8:
            qb, sb = O.quant_weight_block128(w)
        elif fmt == lq.BLOCK_FP8_UE8M0:
            qb, sb = U.quant_weight_block128_ue8m0(w)
        else:
            qb, sb = O.quant_per_channel(w, FMT_NAME[fmt])
        _cache.clear()   # keep one weight in host memory at a time
        _cache[key] = (qb, sb, torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda())
    return _cache[key]


def _check(fmt, M, N, K, n_cols=192, n_rows=None, stripes=False):
    """The table's variant at full size against the oracle on sampled
    outputs: n_cols random columns on every row (or n_rows random rows), and
    with `stripes` also every row of 16-column stripes at the first output
    tile, across the boundary of the first two tiles and at the last tile."""
    qb, sb, B, b_s = _weights(fmt, N, K)
    x = inputs.activations(M, K, seed=inputs.stable_seed("full-A", fmt, M, N, K)).float().numpy()
    block = fmt in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0)
    if fmt == lq.BLOCK_FP8:
        qa, sa = O.quant_per_token_group128(x)
    elif fmt == lq.BLOCK_FP8_UE8M0:
        qa, sa = U.quant_per_token_group128_ue8m0(x)
    else:
        qa, sa = O.quant_per_token(x, FMT_NAME[fmt])
    C = lq.scaled_mm(fmt, torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(), B, b_s)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    v = lq.select_variant(fmt, M, N, K)
    got_all = C.float().cpu().numpy().astype(np.float64)
    sa_f = U.e8m0_decode(sa) if fmt == lq.BLOCK_FP8_UE8M0 else sa
    sb_f = U.e8m0_decode(sb) if fmt == lq.BLOCK_FP8_UE8M0 else sb

    def ref_of(rows, cols):
        if block:
            return np.stack([O.blockwise_ref(qa[rows], sa_f[rows], qb[n:n + 1], sb_f[n // 128:n // 128 + 1])[:, 0]
                             for n in cols], axis=1)
        return O.scaled_mm_ref(FMT_NAME[fmt], qa[rows], sa[rows], qb[cols], sb[cols])

    rng = np.random.default_rng(M * 1000003 + N + K)
    cols = np.sort(rng.choice(N, size=min(n_cols, N), replace=False))
    rows = np.arange(M) if n_rows is None else np.sort(rng.choice(M, size=n_rows, replace=False))
    assert_close(got_all[np.ix_(rows, cols)], ref_of(rows, cols), f"fmt={fmt} M={M} N={N} K={K} {v.as_dict()}")
    if stripes:
        tn = v.tile_n if not v.swap_ab else 128     # the width of an output tile along N
        all_rows = np.arange(M)
        for lo in (0, tn - 8, N - 16):
            sc = np.arange(lo, lo + 16)
            assert_close(got_all[np.ix_(all_rows, sc)], ref_of(all_rows, sc),
                         f"stripe [{lo}, {lo + 16}) fmt={fmt} M={M} {v.as_dict()}")


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8], ids=["fp8", "int8"])
@pytest.mark.parametrize("layer", list(inputs.QWEN3_8B))
def test_qwen3_8b_decode(cuda_device, fmt, layer):
    K, N = inputs.QWEN3_8B[layer]
    for M in inputs.DECODE_M:
        _check(fmt, M, N, K)


@pytest.mark.parametrize("layer", list(inputs.QWEN3_32B))
def test_qwen3_32b_block_decode(cuda_device, layer):
    K, N = inputs.QWEN3_32B[layer]
    for M in (1, 8, 24, 32):
        _check(lq.BLOCK_FP8, M, N, K, n_cols=96)


@pytest.mark.parametrize("layer", list(inputs.QWEN3_32B))
def test_qwen3_32b_ue8m0_decode(cuda_device, layer):
    K, N = inputs.QWEN3_32B[layer]
    for M in (1, 16, 32):
        _check(lq.BLOCK_FP8_UE8M0, M, N, K, n_cols=96)


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8, lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0],
                         ids=["fp8", "int8", "block", "ue8m0"])
@pytest.mark.parametrize("layer", ["gate_up", "down"])
def test_qwen3_32b_prefill(cuda_device, fmt, layer):
    """M = 256 and 2048 in the table's (persistent, tile 256, Split-K ...)
    launch configuration, sampled outputs plus full-column stripes."""
    K, N = inputs.QWEN3_32B[layer]
    for M in (256, 2048):
        _check(fmt, M, N, K, n_cols=64, n_rows=48, stripes=True)
