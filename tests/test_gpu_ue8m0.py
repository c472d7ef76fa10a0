"""GPU parity of Block_FP8 with UE8M0 scales, through the C ABI: the
quantizers' codes and scale bytes bit-exact against the oracle; the GEMM,
which hands the power-of-two scales to the tensor core's block-scaled MMA,
within tolerance of the oracle (and of the fp32-scale Block_FP8 GEMM given
the same decoded scales), reproducible run to run and identical bit for bit
across the three Split-K reductions."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from oracle import ue8m0_oracle as U
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import bf16_to_f64, wide_range_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(1, 128), (5, 384), (32, 5120), (3, 25600), (257, 1024)])
def test_group128_ue8m0_bitexact(cuda_device, M, K):
    x = inputs.activations(M, K, seed=M * 31 + K)
    q, b = lq.quant_per_token_group128_ue8m0(x.cuda())
    torch.cuda.synchronize()
    q_ref, b_ref = U.quant_per_token_group128_ue8m0(x.float().numpy())
    assert np.array_equal(b.cpu().numpy(), b_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_group128_ue8m0_wide_range_and_zero_groups(cuda_device):
    x = wide_range_rows(1024, seed=8)
    x[0, :128] = 0
    q, b = lq.quant_per_token_group128_ue8m0(x.cuda())
    torch.cuda.synchronize()
    q_ref, b_ref = U.quant_per_token_group128_ue8m0(x.float().numpy())
    assert np.array_equal(b.cpu().numpy(), b_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (1024, 2048)])
def test_weight_block128_ue8m0_bitexact(cuda_device, N, K):
    w = inputs.weights(N, K, seed=N + K + 1)
    q, b = lq.quant_weight_block128_ue8m0(w.cuda())
    torch.cuda.synchronize()
    q_ref, b_ref = U.quant_weight_block128_ue8m0(w.float().numpy())
    assert np.array_equal(b.cpu().numpy(), b_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


VARIANTS = [None,
            dict(swap_ab=0, tile_n=256, split_k=1, stages=3),
            dict(swap_ab=0, tile_n=256, split_k=4, stages=2, reduce=2),
            dict(swap_ab=0, tile_n=128, split_k=1, stages=4),
            dict(swap_ab=0, tile_n=64, split_k=4, stages=3, reduce=2),
            dict(swap_ab=0, tile_n=128, split_k=2, stages=4, reduce=0),
            dict(swap_ab=1, tile_n=16, split_k=8, stages=4, reduce=2),
            dict(swap_ab=1, tile_n=32, split_k=2, stages=3, reduce=1),
            dict(swap_ab=1, tile_n=64, split_k=1, stages=2)]


def _vid(v):
    return "table" if v is None else f"swap{v['swap_ab']}-tn{v['tile_n']}-s{v['split_k']}-r{v.get('reduce', 1)}"


@pytest.mark.parametrize("vd", VARIANTS, ids=_vid)
@pytest.mark.parametrize("M,N,K", [(1, 256, 1024), (24, 384, 2048), (200, 512, 1152)])
def test_blockwise_ue8m0_gemm(cuda_device, vd, M, N, K):
    x = inputs.activations(M, K, seed=M + N + K)
    w = inputs.weights(N, K, seed=N * K)
    qa, ba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    qb, bb = U.quant_weight_block128_ue8m0(w.float().numpy())
    A, BA, B, BB = (torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (qa, ba, qb, bb))
    v = None if vd is None else lq.make_variant(**vd)
    C = lq.scaled_mm("block_fp8_ue8m0", A, BA, B, BB, variant=v)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    ref = U.blockwise_ue8m0_ref(qa, ba, qb, bb)
    ok, worst = O.within_tolerance(bf16_to_f64(C), ref, rms_of=ref)
    assert ok, worst
    # run to run: the same bits
    C2 = lq.scaled_mm("block_fp8_ue8m0", A, BA, B, BB, variant=v)
    torch.cuda.synchronize()
    assert torch.equal(C, C2)
    # the fp32-scale Block_FP8 GEMM (per-block promotion) given the decoded
    # scales computes the same product: within tolerance of the oracle too
    if vd is None or vd["swap_ab"] or vd["tile_n"] <= 128:
        sa32 = torch.from_numpy(U.e8m0_decode(ba).astype(np.float32)).cuda()
        sb32 = torch.from_numpy(U.e8m0_decode(bb).astype(np.float32)).cuda()
        C32 = lq.scaled_mm("block_fp8", A, sa32, B, sb32, variant=v)
        torch.cuda.synchronize()
        ok, worst = O.within_tolerance(bf16_to_f64(C32), ref, rms_of=ref)
        assert ok, worst


@pytest.mark.parametrize("swap,tn", [(1, 16), (1, 32), (1, 64), (0, 64), (0, 128), (0, 256)])
def test_ue8m0_reduce_modes_bitwise_identical(cuda_device, swap, tn):
    """Separate kernel, last arriver and cluster reduction sum the same
    partials (each already carrying its block scales) in the same order."""
    M, N, K = 40, 512, 2304
    x = inputs.activations(M, K, seed=61)
    w = inputs.weights(N, K, seed=62)
    qa, ba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    qb, bb = U.quant_weight_block128_ue8m0(w.float().numpy())
    A, BA, B, BB = (torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (qa, ba, qb, bb))
    ref = U.blockwise_ue8m0_ref(qa, ba, qb, bb)
    for S in (2, 4, 8, 16):
        outs = []
        for red in (0, 1, 2):
            v = lq.make_variant(swap_ab=swap, tile_n=tn, split_k=S, stages=2, reduce=red)
            lq.reserve_workspace(0, lq.workspace_bytes("block_fp8_ue8m0", M, N, K, v))
            outs.append(lq.scaled_mm("block_fp8_ue8m0", A, BA, B, BB, variant=v).clone())
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2]), f"S={S}"
        ok, worst = O.within_tolerance(bf16_to_f64(outs[2]), ref, rms_of=ref)
        assert ok, (S, worst)
    assert lq.device_status(0) == 0


@pytest.mark.parametrize("vd", [dict(swap_ab=0, tile_n=256, split_k=1), dict(swap_ab=0, tile_n=128, split_k=2),
                                dict(swap_ab=1, tile_n=16, split_k=8, reduce=2), None], ids=_vid)
def test_ue8m0_exponent_range(cuda_device, vd):
    """Activation rows scaled by 2^-100 .. 2^90 (scale bytes from about 19 to
    235) and an all-zero 128-group (byte 0, 2^-127): the tensor core applies
    2^(ea + eb) exactly over that range; every row within tolerance of its
    own rms (the rows differ by 2^190)."""
    M, N, K = 10, 256, 1024
    x = inputs.activations(M, K, seed=71).float()
    ks = [-100, -60, -20, 0, 30, 60, 90, -100, 45, 0]
    x = x * torch.tensor([2.0 ** k for k in ks])[:, None]
    x[3, 256:384] = 0
    x = x.to(torch.bfloat16)
    w = inputs.weights(N, K, seed=72)
    qa, ba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    qb, bb = U.quant_weight_block128_ue8m0(w.float().numpy())
    assert ba.min() == 0 and ba.max() >= 200
    A, BA, B, BB = (torch.from_numpy(np.ascontiguousarray(t)).cuda() for t in (qa, ba, qb, bb))
    v = None if vd is None else lq.make_variant(**vd)
    C = lq.scaled_mm("block_fp8_ue8m0", A, BA, B, BB, variant=v)
    torch.cuda.synchronize()
    ref = U.blockwise_ue8m0_ref(qa, ba, qb, bb)
    got = bf16_to_f64(C)
    for m in range(M):
        ok, worst = O.within_tolerance(got[m:m + 1], ref[m:m + 1], rms_of=ref[m:m + 1])
        assert ok, (m, ks[m], worst)


def test_ue8m0_deep_k_sampled(cuda_device):
    """K = 25600 (Qwen3-32B down, 200 scale groups) in the prefill tile and
    the decode tile, on sampled output columns against the oracle."""
    M, N, K = 64, 512, 25600
    x = inputs.activations(M, K, seed=81)
    w = inputs.weights(N, K, seed=82)
    qa, ba = lq.quant_per_token_group128_ue8m0(x.cuda())
    qb, bb = lq.quant_weight_block128_ue8m0(w.cuda())
    cols = np.array([0, 1, 127, 128, 300, 511])
    ra, rba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    rb, rbb = U.quant_weight_block128_ue8m0(w.float().numpy())
    ref = np.stack([U.blockwise_ue8m0_ref(ra, rba, rb[n:n + 1], rbb[n // 128:n // 128 + 1])[:, 0] for n in cols], 1)
    for v in (lq.make_variant(swap_ab=0, tile_n=256, split_k=1), lq.make_variant(swap_ab=0, tile_n=128, split_k=4),
              lq.make_variant(swap_ab=1, tile_n=16, split_k=8, reduce=2)):
        C = lq.scaled_mm("block_fp8_ue8m0", qa, ba, qb, bb, variant=v)
        torch.cuda.synchronize()
        ok, worst = O.within_tolerance(bf16_to_f64(C)[:, cols], ref)
        assert ok, (v.as_dict(), worst)


def test_ue8m0_end_to_end_from_bf16(cuda_device):
    """bf16 activations and weights -> the library's own UE8M0 quantizers ->
    the GEMM, against the oracle's product of the oracle's codes."""
    M, N, K = 16, 1024, 4096
    x = inputs.activations(M, K, seed=51)
    w = inputs.weights(N, K, seed=52)
    qa, ba = lq.quant_per_token_group128_ue8m0(x.cuda())
    qb, bb = lq.quant_weight_block128_ue8m0(w.cuda())
    C = lq.scaled_mm("block_fp8_ue8m0", qa, ba, qb, bb)
    torch.cuda.synchronize()
    ra, rba = U.quant_per_token_group128_ue8m0(x.float().numpy())
    rb, rbb = U.quant_weight_block128_ue8m0(w.float().numpy())
    ref = U.blockwise_ue8m0_ref(ra, rba, rb, rbb)
    ok, worst = O.within_tolerance(bf16_to_f64(C), ref, rms_of=ref)
    assert ok, worst
