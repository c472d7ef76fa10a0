"""Failure detection on the GPU without a fault: a test hook leaves one K tile
of every CTA unloaded, so the tensor-core warp's bounded wait runs out.  The
kernel must report it through the device status word (LQ_ERR_DEVICE_TIMEOUT),
release its resources and return, and the context must stay usable."""

import pytest
import torch

from quantized_linear_gemm_b200 import lq

from _lqtest import assert_close, make_problem

pytestmark = pytest.mark.gpu

TIMEOUT = 6
CASES = [
    (lq.FP8_DYNAMIC, dict(swap_ab=1, tile_n=16, split_k=1, stages=2)),
    (lq.W8A8_INT8, dict(swap_ab=0, tile_n=128, split_k=1, stages=3)),
    (lq.FP8_DYNAMIC, dict(swap_ab=1, tile_n=32, split_k=4, stages=2, reduce=0)),
    (lq.FP8_DYNAMIC, dict(swap_ab=1, tile_n=16, split_k=4, stages=2, reduce=1)),
    (lq.W8A8_INT8, dict(swap_ab=1, tile_n=16, split_k=4, stages=2, reduce=2)),      # cluster, push
    (lq.FP8_DYNAMIC, dict(swap_ab=0, tile_n=128, split_k=2, stages=3, reduce=2)),   # cluster, pull
    (lq.BLOCK_FP8, dict(swap_ab=1, tile_n=16, split_k=2, stages=2, reduce=2)),
    (lq.FP8_DYNAMIC, dict(swap_ab=0, tile_n=64, split_k=1, stages=3, persistent=1)),   # persistent CTAs
    (lq.BLOCK_FP8_UE8M0, dict(swap_ab=0, tile_n=128, split_k=1, stages=3)),            # block-scaled MMA
]


@pytest.mark.parametrize("fmt,vd", CASES, ids=[f"{f}-{i}" for i, (f, _) in enumerate(CASES)])
def test_bounded_wait_runs_out_and_is_reported(cuda_device, fmt, vd):
    prob = make_problem(fmt, 24, 384, 1152, seed=300)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(**vd)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, 24, 384, 1152, v))
    assert lq.device_status(0) == 0
    lq.test_inject_stall(1, 200_000_000)            # K tile 1 never arrives; waits give up after 0.2 s
    try:
        lq.scaled_mm(fmt, A, sa, B, sb, variant=v)
        torch.cuda.synchronize()                     # the kernel returned: nothing hung
        assert lq.device_status(0) == TIMEOUT
    finally:
        lq.test_inject_stall(-1, 0)
    # the context is intact: the same call now gives the oracle's result
    C = lq.scaled_mm(fmt, A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert_close(C, prob.reference(), "after a timed-out launch")
