"""lq_scaled_mm_noalloc: the entry point for callers that cannot allocate
device memory when they run a GEMM (code inside a CUDA-graph capture with the
global capture mode, frameworks that hand out memory only through their own
pool, services that must not allocate after start-up).  Its Split-K partials
live in a fixed array that the library reserves in device memory, so it must
give the same results as lq_scaled_mm.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes alone in a fresh
process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import lq

from _lqtest import bf16_to_f64, make_problem

WORKSPACE = 4        # LQ_ERR_WORKSPACE
SCRATCH_BYTES = 16 << 20


def test_rejects_partials_beyond_the_fixed_array():
    """A Split-K call whose partials do not fit in 16 MiB is refused before
    anything is launched (no GPU needed to check this)."""
    v = lq.make_variant(swap_ab=1, tile_n=32, split_k=8, reduce=0)
    M, N, K = 32, 51200, 5120                           # 8 * 32 * 51200 * 4 B = 52 MB
    assert 8 * M * N * 4 > SCRATCH_BYTES
    fake = 0x10000
    rc = lq.lib().lq_scaled_mm_noalloc(0, fake, fake, fake, fake, fake, M, N, K, v, None)
    assert rc == WORKSPACE


CASES = [
    # (fmt, M, N, K, variant)
    (lq.FP8_DYNAMIC, 8, 4096, 4096, dict(swap_ab=1, tile_n=16, split_k=8, stages=4)),
    (lq.W8A8_INT8, 24, 6144, 4096, dict(swap_ab=1, tile_n=32, split_k=4, stages=4)),
    (lq.BLOCK_FP8, 5, 5120, 8192, dict(swap_ab=1, tile_n=16, split_k=8, stages=2)),
    (lq.FP8_DYNAMIC, 96, 1024, 2048, dict(swap_ab=0, tile_n=128, split_k=2, stages=4)),
]


@pytest.mark.gpu
def test_noalloc_matches_scaled_mm_on_two_calls_in_a_row(cuda_device):
    """Two calls in a row of the allocation-free entry point (the second one
    reuses the fixed array the first one filled) each give the output of
    lq_scaled_mm with the same variant, within the suite's tolerance, and the
    oracle's result within the same tolerance."""
    probs = [make_problem(fmt, M, N, K, seed=100 + i) for i, (fmt, M, N, K, _) in enumerate(CASES)]
    dev_inputs = [p.device() for p in probs]
    for first, second in ((0, 1), (2, 3), (1, 0)):
        outs = []
        for idx in (first, second):                    # two calls in a row, nothing in between
            fmt, M, N, K, vd = CASES[idx]
            A, sa, B, sb = dev_inputs[idx]
            outs.append(lq.scaled_mm_noalloc(fmt, A, sa, B, sb, variant=lq.make_variant(**vd)))
        torch.cuda.synchronize()
        for idx, C_noalloc in zip((first, second), outs):
            fmt, M, N, K, vd = CASES[idx]
            A, sa, B, sb = dev_inputs[idx]
            C_ref = lq.scaled_mm(fmt, A, sa, B, sb, variant=lq.make_variant(**dict(vd, reduce=0)))
            torch.cuda.synchronize()
            got, want = bf16_to_f64(C_noalloc), bf16_to_f64(C_ref)
            ok, worst = O.within_tolerance(got, want)
            assert ok, f"case {idx}: differs from lq_scaled_mm, worst ratio {worst:.3g}"
            ok, worst = O.within_tolerance(got, probs[idx].reference())
            assert ok, f"case {idx}: outside the oracle tolerance, worst ratio {worst:.3g}"
            # same kernels, same fixed reduction order: the bits agree too
            assert np.array_equal(got, want), f"case {idx}: not bit-identical to lq_scaled_mm"


@pytest.mark.gpu
def test_noalloc_without_split_and_with_table_variant(cuda_device):
    """split_k = 1 (no scratch needed) and variant = NULL also work."""
    for i, (fmt, M, N, K, _) in enumerate(CASES[:2]):
        A, sa, B, sb = make_problem(fmt, M, N, K, seed=200 + i).device()
        for v in (lq.make_variant(swap_ab=1, tile_n=32, split_k=1), None):
            C = lq.scaled_mm_noalloc(fmt, A, sa, B, sb, variant=v)
            C_ref = lq.scaled_mm(fmt, A, sa, B, sb, variant=v if v is not None else None)
            torch.cuda.synchronize()
            assert O.within_tolerance(bf16_to_f64(C), bf16_to_f64(C_ref))[0]
