"""GPU tests of the boundary's contracts around the GEMM: a default (NULL)
variant is safe right after a weight is quantized on the same stream, also
inside one CUDA graph; a captured Split-K graph stays valid after a later
call grows the workspace; lq_quant_scaled_mm runs the caller's variant
unchanged on its two-kernel path.  Every result is compared with the oracle."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import assert_close, make_problem

pytestmark = pytest.mark.gpu


def _capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


@pytest.mark.parametrize("fmt,M,N,K", [("fp8_dynamic", 8, 6144, 4096),      # Qwen3-8B qkv
                                       ("w8a8_int8", 24, 4096, 12288),      # Qwen3-8B down
                                       ("block_fp8", 8, 5120, 8192)])       # Qwen3-32B o
def test_default_variant_after_weight_quantization_in_one_graph(cuda_device, fmt, M, N, K):
    """Weight quantization, activation quantization and lq_scaled_mm with
    variant NULL captured in one graph on one stream.  Between replays the
    bf16 weight changes, so a GEMM that read B before the weight quantizer
    had finished would return the previous replay's product."""
    prev = lq.declare_static_weights(False)
    try:
        lq.init_device(0)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        w_dev = inputs.weights(N, K, seed=101).cuda()
        x_dev = inputs.activations(M, K, seed=102).cuda()
        code_dt = torch.int8 if fmt == "w8a8_int8" else torch.uint8
        block = fmt == "block_fp8"
        qb = torch.empty((N, K), dtype=code_dt, device="cuda")
        sb = torch.empty((N // 128, K // 128) if block else (N,), dtype=torch.float32, device="cuda")
        qa = torch.empty((M, K), dtype=code_dt, device="cuda")
        sa = torch.empty((M, K // 128) if block else (M,), dtype=torch.float32, device="cuda")
        C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")

        def step():
            if block:
                lq.quant_weight_block128(w_dev, qb, sb, stream=s)
                lq.quant_per_token_group128(x_dev, qa, sa, stream=s)
            else:
                lq.quant_per_token(fmt, w_dev, qb, sb, stream=s)
                lq.quant_per_token(fmt, x_dev, qa, sa, stream=s)
            lq.scaled_mm(fmt, qa, sa, qb, sb, C=C, stream=s)   # variant NULL

        g = _capture(step, s)
        xn = x_dev.float().cpu().numpy()
        for seed in (103, 104, 105):
            w = inputs.weights(N, K, seed=seed)
            w_dev.copy_(w)
            torch.cuda.synchronize()
            with torch.cuda.stream(s):
                g.replay()
            torch.cuda.synchronize()
            wn = w.float().numpy()
            if block:
                ra, rsa = O.quant_per_token_group128(xn)
                rb, rsb = O.quant_weight_block128(wn)
                ref = O.blockwise_ref(ra, rsa, rb, rsb)
            else:
                ra, rsa = O.quant_per_token(xn, fmt)
                rb, rsb = O.quant_per_channel(wn, fmt)
                ref = O.scaled_mm_ref(fmt, ra, rsa, rb, rsb)
            assert_close(C, ref, f"{fmt} replay with weight seed {seed}")
        del g
        assert lq.device_status(0) == 0
    finally:
        lq.declare_static_weights(prev)


@pytest.mark.parametrize("reduce", [0, 1])
def test_workspace_growth_keeps_an_earlier_graph_valid(cuda_device, reduce):
    """Capture a Split-K call that uses the workspace, then make a much larger
    Split-K call eagerly (the workspace grows), then replay the graph: the
    replaced workspace was kept, so the replay is still correct."""
    fmt = lq.FP8_DYNAMIC
    small = make_problem(fmt, 16, 512, 2048, seed=111)
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=8, reduce=reduce)
    lq.init_device(0)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, 16, 512, 2048, v))
    A, sa, B, sb = small.device()
    out = torch.empty((16, 512), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = _capture(lambda: lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=v, stream=s), s)
    # a call whose partials need far more than the reserved workspace
    big = make_problem(fmt, 256, 4096, 4096, seed=112, outliers=False)
    vb = lq.make_variant(swap_ab=0, tile_n=128, split_k=16, reduce=reduce)
    need = lq.workspace_bytes(fmt, 256, 4096, 4096, vb)
    assert need > 64 * lq.workspace_bytes(fmt, 16, 512, 2048, v)
    Ab, sab, Bb, sbb = big.device()
    Cb = lq.scaled_mm(fmt, Ab, sab, Bb, sbb, variant=vb)
    torch.cuda.synchronize()
    assert_close(Cb, big.reference(), "the growing call")
    for _ in range(2):
        out.zero_()
        with torch.cuda.stream(s):
            g.replay()
        torch.cuda.synchronize()
        assert_close(out, small.reference(), "replay after growth")
    del g
    assert lq.device_status(0) == 0


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
@pytest.mark.parametrize("reduce", [0, 1])
def test_quant_scaled_mm_runs_the_callers_variant(cuda_device, fmt, reduce):
    """split_k 32 with a workspace reduction (the cluster reduction allows at
    most 16) through lq_quant_scaled_mm under the default fusion limit: the
    two kernels run with that variant and give the codes, scales and C of
    lq_quant_per_token followed by lq_scaled_mm."""
    M, N, K = 8, 1024, 8192
    x = inputs.activations(M, K, seed=121).cuda()
    w = inputs.weights(N, K, seed=122)
    qb, sb = lq.quant_per_token(fmt, w.cuda())
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=32, reduce=reduce)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, M, N, K, v))
    C, q, s_ = lq.quant_scaled_mm(fmt, x, qb, sb, variant=v)
    qa2, sa2 = lq.quant_per_token(fmt, x)
    C2 = lq.scaled_mm(fmt, qa2, sa2, qb, sb, variant=v)
    torch.cuda.synchronize()
    assert torch.equal(q, qa2) and torch.equal(s_, sa2) and torch.equal(C, C2)
    ra, rsa = O.quant_per_token(x.float().cpu().numpy(), fmt)
    rb, rsb = O.quant_per_channel(w.float().numpy(), fmt)
    assert np.array_equal(q.cpu().numpy(), ra)
    assert_close(C, O.scaled_mm_ref(fmt, ra, rsa, rb, rsb), f"{fmt} split 32 reduce {reduce}")
    assert lq.device_status(0) == 0
