"""GPU parity of the bias epilogue (lq_scaled_mm_bias) in every output path
(Standard / Swap-AB stores, the three Split-K reductions, Block_FP8 with fp32
and UE8M0 scales), and of one rank's slice of the N-sliced linear."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq, parallel

from _lqtest import FMT_NAME, assert_close, make_problem

pytestmark = pytest.mark.gpu

VARIANTS = [dict(swap_ab=0, tile_n=128, split_k=1, stages=4),
            dict(swap_ab=0, tile_n=64, split_k=4, stages=3, reduce=0),
            dict(swap_ab=0, tile_n=128, split_k=2, stages=4, reduce=1),
            dict(swap_ab=0, tile_n=128, split_k=4, stages=3, reduce=2),
            dict(swap_ab=1, tile_n=16, split_k=1, stages=4),
            dict(swap_ab=1, tile_n=16, split_k=8, stages=4, reduce=2),
            dict(swap_ab=1, tile_n=32, split_k=4, stages=3, reduce=1),
            dict(swap_ab=1, tile_n=64, split_k=2, stages=2, reduce=0)]


def _vid(v):
    return f"swap{v['swap_ab']}-tn{v['tile_n']}-s{v['split_k']}-r{v.get('reduce', 1)}"


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8, lq.BLOCK_FP8], ids=["fp8", "int8", "block"])
@pytest.mark.parametrize("vd", VARIANTS, ids=_vid)
def test_bias_every_path(cuda_device, fmt, vd):
    M, N, K = 40, 384, 1024
    prob = make_problem(fmt, M, N, K, seed=7)
    A, sa, B, sb = prob.device()
    bias = torch.from_numpy(np.random.default_rng(8).standard_normal(N) * 4).to(torch.bfloat16).cuda()
    v = lq.make_variant(**vd)
    C = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=v)
    torch.cuda.synchronize()
    ref = prob.reference() + bias.double().cpu().numpy()[None, :]
    assert_close(C, ref, f"bias {FMT_NAME[fmt]} {vd}")
    # a zero bias gives lq_scaled_mm's output
    C0 = lq.scaled_mm_bias(fmt, A, sa, B, sb, torch.zeros_like(bias), variant=v)
    C1 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert torch.equal(C0, C1)


def test_bias_ue8m0(cuda_device):
    from oracle import ue8m0_oracle as U
    M, N, K = 16, 256, 1024
    x = inputs.activations(M, K, seed=9)
    w = inputs.weights(N, K, seed=10)
    qa, ba = lq.quant_per_token_group128_ue8m0(x.cuda())
    qb, bb = lq.quant_weight_block128_ue8m0(w.cuda())
    bias = torch.linspace(-3, 3, N).to(torch.bfloat16).cuda()
    C = lq.scaled_mm_bias("block_fp8_ue8m0", qa, ba, qb, bb, bias)
    torch.cuda.synchronize()
    ra, rba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    rb, rbb = U.quant_weight_block128_ue8m0(w.float().numpy())
    ref = U.blockwise_ue8m0_ref(ra, rba, rb, rbb) + bias.double().cpu().numpy()[None, :]
    assert_close(C, ref, "bias ue8m0")


def test_column_parallel_slice_matches_full_layer(cuda_device):
    """Rank r's slice of an N-sliced linear gives columns [n0, n1) of the
    full layer (same variant: the same bits)."""
    M, N, K = 8, 1024, 2048
    prob = make_problem(lq.FP8_DYNAMIC, M, N, K, seed=11)
    A, sa, B, sb = prob.device()
    bias = torch.from_numpy(np.random.default_rng(12).standard_normal(N)).to(torch.bfloat16).cuda()
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=4, stages=4, reduce=2)
    full = lq.scaled_mm_bias("fp8_dynamic", A, sa, B, sb, bias, variant=v)
    for rank in range(4):
        layer = parallel.ColumnParallelLinear.from_full("fp8_dynamic", B, sb, bias, rank, 4)
        C = lq.scaled_mm_bias("fp8_dynamic", A, sa, layer.B, layer.b_scales, layer.bias, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(C, full[:, layer.n0:layer.n1])
        # the layer's own call (the dispatch table's variant for the slice's N)
        Cl = layer.forward(A, sa, gather=False)
        torch.cuda.synchronize()
        ref = prob.reference(cols=slice(layer.n0, layer.n1)) + bias.double().cpu().numpy()[None, layer.n0:layer.n1]
        assert_close(Cl, ref, f"slice {rank}", rms_of=ref)
