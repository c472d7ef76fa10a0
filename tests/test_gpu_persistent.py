"""GPU parity of the persistent scaled_mm (one CTA per SM looping over output
tiles, two tensor-memory accumulators), through the C ABI: the same bits as
the one-tile-per-CTA kernel with the same tile, within tolerance of the
oracle, exact INT8 accumulators, bias, ragged tails, several tiles per CTA,
and graph replay."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import assert_close, make_problem

pytestmark = pytest.mark.gpu

FMTS = [lq.FP8_DYNAMIC, lq.W8A8_INT8]
FMT_IDS = ["fp8", "int8"]


def _pair(prob, tn, stages=0, pdl=1, bias=None):
    """(persistent C, one-tile-per-CTA C) for the same tile."""
    A, sa, B, sb = prob.device()
    outs = []
    for pers in (1, 0):
        v = lq.make_variant(swap_ab=0, tile_n=tn, split_k=1, stages=stages, pdl=pdl, persistent=pers)
        if bias is None:
            outs.append(lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v))
        else:
            outs.append(lq.scaled_mm_bias(prob.fmt, A, sa, B, sb, bias, variant=v))
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    return outs


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [64, 128, 256])
@pytest.mark.parametrize("stages", [2, 3, 0])
def test_persistent_small_ragged(cuda_device, fmt, tn, stages):
    """M = 300 (a ragged m-block), N = 1000 (ragged n-block), K = 1040 (a
    16-wide last K tile): fewer tiles than SMs, one tile per CTA."""
    prob = make_problem(fmt, 300, 1000, 1040, seed=401)
    Cp, Cs = _pair(prob, tn, stages)
    assert torch.equal(Cp, Cs)
    assert_close(Cp, prob.reference(), f"persistent tn={tn} stages={stages}")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [64, 128, 256])
@pytest.mark.parametrize("pdl", [0, 1, 2])
def test_persistent_many_tiles_per_cta(cuda_device, fmt, tn, pdl):
    """M = 1100, N = 4096: 9 x (64 .. 16) tiles, up to four per CTA, both
    accumulator buffers reused; equal to the one-tile kernel bit for bit and
    to the oracle on sampled rows and columns (every m-block, both ends)."""
    M, N, K = 1100, 4096, 1024
    prob = make_problem(fmt, M, N, K, seed=402 + tn, outliers=False)
    Cp, Cs = _pair(prob, tn, pdl=pdl)
    assert torch.equal(Cp, Cs)
    rows = np.array([0, 127, 128, 500, 1023, 1024, 1099])
    cols = np.array([0, 7, 255, 256, 2047, 4088, 4095])
    ref = O.scaled_mm_ref({lq.FP8_DYNAMIC: O.FMT_FP8_DYNAMIC, lq.W8A8_INT8: O.FMT_W8A8_INT8}[fmt],
                          prob.qa[rows], prob.sa[rows], prob.qb[cols], prob.sb[cols])
    got = Cp.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)]
    ok, worst = O.within_tolerance(got, ref)
    assert ok, worst


def test_persistent_int8_accumulators_exact(cuda_device):
    prob = make_problem(lq.W8A8_INT8, 300, 768, 1152, seed=403)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=256, split_k=1, persistent=1)
    C, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.acc_exact(O.FMT_W8A8_INT8, prob.qa, prob.qb))
    assert_close(C, prob.reference(), "int8 persistent C")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
def test_persistent_bias(cuda_device, fmt):
    prob = make_problem(fmt, 260, 512, 1024, seed=404)
    g = torch.Generator().manual_seed(405)
    bias = (torch.randn(512, generator=g) * 0.5).to(torch.bfloat16)
    Cp, Cs = _pair(prob, 128, bias=bias.cuda())
    assert torch.equal(Cp, Cs)
    ref = prob.reference() + bias.double().numpy()[None, :]
    assert_close(Cp, ref, "persistent bias")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
def test_persistent_graph_replay_and_default(cuda_device, fmt):
    """Bitwise reproducible under CUDA-graph replay; the default variant for a
    many-tile Standard shape outside the table (at least two tiles per SM) is
    the persistent one."""
    M, N, K = 2048, 8192, 512
    prob = make_problem(fmt, M, N, K, seed=406, outliers=False)
    A, sa, B, sb = prob.device()
    v = lq.select_variant(fmt, M, N, K)
    assert v.persistent == 1 and v.swap_ab == 0 and v.split_k == 1
    C0 = lq.scaled_mm(fmt, A, sa, B, sb).clone()
    out = torch.empty_like(C0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(2):
                lq.scaled_mm(fmt, A, sa, B, sb, C=out, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C0)
    del g
    rows = np.arange(0, M, 97)
    cols = np.arange(0, N, 331)
    name = {lq.FP8_DYNAMIC: O.FMT_FP8_DYNAMIC, lq.W8A8_INT8: O.FMT_W8A8_INT8}[fmt]
    ref = O.scaled_mm_ref(name, prob.qa[rows], prob.sa[rows], prob.qb[cols], prob.sb[cols])
    ok, worst = O.within_tolerance(C0.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)], ref)
    assert ok, worst
    assert lq.device_status(0) == 0


def test_persistent_refuses_what_it_does_not_do(cuda_device):
    prob = make_problem(lq.FP8_DYNAMIC, 64, 256, 512, seed=407)
    A, sa, B, sb = prob.device()
    for bad in (dict(swap_ab=1, tile_n=16, persistent=1), dict(swap_ab=0, tile_n=128, split_k=2, persistent=1),
                dict(swap_ab=0, tile_n=128, persistent=4)):
        with pytest.raises(lq.LQError):
            lq.scaled_mm(lq.FP8_DYNAMIC, A, sa, B, sb, variant=lq.make_variant(**bad))
    qa = torch.zeros((64, 512), dtype=torch.uint8, device="cuda")
    with pytest.raises(lq.LQError):
        lq.scaled_mm("block_fp8", qa, torch.ones((64, 4), device="cuda"), torch.zeros((256, 512), dtype=torch.uint8,
                     device="cuda"), torch.ones((2, 4), device="cuda"),
                     variant=lq.make_variant(swap_ab=0, tile_n=128, persistent=1))


# ----------------------------------------------------------- CTA pairs (persistent = 2)
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [128, 256])
def test_pair_small_ragged(cuda_device, fmt, tn):
    """CTA pairs (tcgen05 cta_group::2, 256-row tiles): M = 300 (the second
    CTA's rows partly past M), N = 1000 (ragged), K = 1040 (ragged K tile):
    within tolerance of the oracle and bitwise reproducible."""
    prob = make_problem(fmt, 300, 1000, 1040, seed=411)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=tn, split_k=1, persistent=2)
    C0 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v).clone()
    C1 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert torch.equal(C0, C1)
    assert_close(C0, prob.reference(), f"pair tn={tn}")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [128, 256])
def test_pair_many_tiles_equals_one_sm(cuda_device, fmt, tn):
    """M = 1100, N = 4096: several 256-row tiles per pair, both accumulator
    buffers of both CTAs reused; the same bits as the one-SM persistent kernel
    (each SM's tensor core computes its 128 rows with the same MMA sequence)
    and the oracle on sampled outputs."""
    M, N, K = 1100, 4096, 1024
    prob = make_problem(fmt, M, N, K, seed=412 + tn, outliers=False)
    A, sa, B, sb = prob.device()
    Cp = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=lq.make_variant(swap_ab=0, tile_n=tn, persistent=2))
    C1 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=lq.make_variant(swap_ab=0, tile_n=tn, persistent=1))
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert torch.equal(Cp, C1)
    rows = np.array([0, 127, 128, 255, 256, 700, 1023, 1024, 1099])
    cols = np.array([0, 7, 127, 128, 255, 256, 2047, 4095])
    name = {lq.FP8_DYNAMIC: O.FMT_FP8_DYNAMIC, lq.W8A8_INT8: O.FMT_W8A8_INT8}[fmt]
    ref = O.scaled_mm_ref(name, prob.qa[rows], prob.sa[rows], prob.qb[cols], prob.sb[cols])
    ok, worst = O.within_tolerance(Cp.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)], ref)
    assert ok, worst


def test_pair_int8_exact_bias_and_graph(cuda_device):
    prob = make_problem(lq.W8A8_INT8, 520, 768, 1152, seed=413)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=256, persistent=2)
    C, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.acc_exact(O.FMT_W8A8_INT8, prob.qa, prob.qb))
    assert_close(C, prob.reference(), "pair int8")
    g = torch.Generator().manual_seed(414)
    bias = (torch.randn(768, generator=g) * 0.5).to(torch.bfloat16).cuda()
    Cb = lq.scaled_mm_bias(lq.W8A8_INT8, A, sa, B, sb, bias, variant=v)
    torch.cuda.synchronize()
    assert_close(Cb, prob.reference() + bias.double().cpu().numpy()[None, :], "pair bias")
    out = torch.empty_like(C)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(gr, stream=s):
            lq.scaled_mm(lq.W8A8_INT8, A, sa, B, sb, C=out, variant=v, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        out.zero_()
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C)
    del gr
    assert lq.device_status(0) == 0


# ------------------------------------------------ CTA pairs with Split-K (persistent = 2, reduce 0)
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [128, 256])
def test_pair_split_equals_one_sm_split(cuda_device, fmt, tn):
    """Split s covers the same K blocks in both kernels and the partials are
    summed by the same reduction, so CTA pairs with split 2 and 4 give the
    bits of the one-SM split; ragged M, N and K (K = 1040: a short last K
    tile); M = 1100 with split 4 has more units than pairs."""
    for (M, N, K, S) in ((300, 1000, 1040, 2), (1100, 4096, 1024, 4)):
        prob = make_problem(fmt, M, N, K, seed=430 + S + tn, outliers=False)
        A, sa, B, sb = prob.device()
        vp = lq.make_variant(swap_ab=0, tile_n=tn, split_k=S, reduce=0, persistent=2)
        v1 = lq.make_variant(swap_ab=0, tile_n=tn, split_k=S, reduce=0)
        Cp = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=vp)
        C1 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v1)
        torch.cuda.synchronize()
        assert lq.device_status(0) == 0
        assert torch.equal(Cp, C1), (M, N, K, S)
        if M == 300:
            assert_close(Cp, prob.reference(), f"pair split {S} tn={tn}")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("S", [3, 5, 12])
def test_pair_split_any_count_and_empty_splits(cuda_device, fmt, S):
    """Split counts that are not powers of two, and S = 12 > T = 9 K tiles
    (three splits own no K block and contribute zero partials): within
    tolerance of the oracle, reproducible, and for W8A8_INT8 the exact
    accumulators."""
    prob = make_problem(fmt, 300, 1000, 1040, seed=440 + S)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=256, split_k=S, reduce=0, persistent=2)
    C0 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v).clone()
    C1 = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert torch.equal(C0, C1)
    assert_close(C0, prob.reference(), f"pair split {S}")
    if fmt == lq.W8A8_INT8:
        C2, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(C2, C0)
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.acc_exact(O.FMT_W8A8_INT8, prob.qa, prob.qb))


def test_pair_split_bias_graph_and_noalloc(cuda_device):
    """Bias through the reduction, graph replay of the two launches, and the
    allocation-free entry point (its fixed scratch array) with the same bits."""
    fmt = lq.FP8_DYNAMIC
    prob = make_problem(fmt, 256, 1024, 2560, seed=450)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=256, split_k=3, reduce=0, persistent=2)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, 256, 1024, 2560, v))
    C = lq.scaled_mm(fmt, A, sa, B, sb, variant=v)
    g = torch.Generator().manual_seed(451)
    bias = (torch.randn(1024, generator=g) * 0.5).to(torch.bfloat16).cuda()
    Cb = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=v)
    Cn = lq.scaled_mm_noalloc(fmt, A, sa, B, sb, variant=v)
    torch.cuda.synchronize()
    assert_close(C, prob.reference(), "pair split 3")
    assert_close(Cb, prob.reference() + bias.double().cpu().numpy()[None, :], "pair split bias")
    assert torch.equal(Cn, C)
    out = torch.empty_like(C)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(gr, stream=s):
            lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=v, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        out.zero_()
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C)
    del gr
    assert lq.device_status(0) == 0


# ------------------------------------ fp32-scale Block_FP8 on CTA pairs (persistent = 2, tile_n 128)
def test_block_pair_equals_one_sm(cuda_device):
    """The pair kernel promotes each 128-K block's partial with the one-SM
    kernel's expression (fmaf of the partial and a_s * b_s, in K order), so
    one split and split 2 (same K blocks per split, same reduction) give the
    one-SM kernel's bits; M = 300 leaves the second CTA's rows partly past M,
    M = 1100 gives several tiles per pair and reuses all four accumulator
    buffers; within tolerance of the oracle."""
    fmt = lq.BLOCK_FP8
    for (M, N, K) in ((300, 1024, 1280), (1100, 2048, 1024)):
        prob = make_problem(fmt, M, N, K, seed=460 + M, outliers=(M == 300))
        A, sa, B, sb = prob.device()
        for S in (1, 2):
            vp = lq.make_variant(swap_ab=0, tile_n=128, split_k=S, reduce=0, persistent=2)
            v1 = lq.make_variant(swap_ab=0, tile_n=128, split_k=S, reduce=0)
            Cp = lq.scaled_mm(fmt, A, sa, B, sb, variant=vp)
            C1 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v1)
            torch.cuda.synchronize()
            assert lq.device_status(0) == 0
            assert torch.equal(Cp, C1), (M, N, K, S)
        if M == 300:
            assert_close(Cp, prob.reference(), "block pair")
        else:
            rows = np.array([0, 127, 128, 255, 256, 700, 1023, 1024, 1099])
            cols = np.array([0, 7, 127, 128, 1023, 2047])
            ok, worst = O.within_tolerance(Cp.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)],
                                           prob.reference(rows, cols))
            assert ok, worst


@pytest.mark.parametrize("S", [3, 12])
def test_block_pair_split_counts_bias_and_graph(cuda_device, S):
    """Split 3, and split 12 over T = 10 K blocks (two empty splits): within
    tolerance of the oracle; the bias epilogue (and bias through the
    reduction); a graph replay gives the same bits."""
    fmt = lq.BLOCK_FP8
    prob = make_problem(fmt, 300, 1024, 1280, seed=470 + S)
    A, sa, B, sb = prob.device()
    v1 = lq.make_variant(swap_ab=0, tile_n=128, persistent=2)
    vs = lq.make_variant(swap_ab=0, tile_n=128, split_k=S, reduce=0, persistent=2)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, 300, 1024, 1280, vs))
    C = lq.scaled_mm(fmt, A, sa, B, sb, variant=vs)
    g = torch.Generator().manual_seed(471)
    bias = (torch.randn(1024, generator=g) * 0.5).to(torch.bfloat16).cuda()
    Cb1 = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=v1)
    Cbs = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=vs)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert_close(C, prob.reference(), f"block pair split {S}")
    refb = prob.reference() + bias.double().cpu().numpy()[None, :]
    assert_close(Cb1, refb, "block pair bias")
    assert_close(Cbs, refb, f"block pair split {S} bias")
    out = torch.empty_like(C)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(gr, stream=s):
            lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=vs, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        out.zero_()
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C)
    del gr
    assert lq.device_status(0) == 0


def test_block_pair_refuses_other_tiles(cuda_device):
    fmt = lq.BLOCK_FP8
    prob = make_problem(fmt, 256, 512, 512, seed=480)
    A, sa, B, sb = prob.device()
    for bad in (dict(swap_ab=0, tile_n=256, persistent=2), dict(swap_ab=0, tile_n=128, persistent=1),
                dict(swap_ab=0, tile_n=128, persistent=3)):
        with pytest.raises(lq.LQError):
            lq.scaled_mm(fmt, A, sa, B, sb, variant=lq.make_variant(**bad))
    ue = make_problem(lq.BLOCK_FP8_UE8M0, 256, 512, 512, seed=481)
    A, sa, B, sb = ue.device()
    with pytest.raises(lq.LQError):   # UE8M0 pairs: 256 x 128 tiles
        lq.scaled_mm(lq.BLOCK_FP8_UE8M0, A, sa, B, sb, variant=lq.make_variant(swap_ab=0, tile_n=256, persistent=2))


# ------------------------------------------ UE8M0 Block_FP8 on CTA pairs (persistent = 2, tile_n 128)
def test_ue8m0_pair_against_oracle_and_one_sm(cuda_device):
    """Block-scaled MMA over a CTA pair (each CTA's tensor memory holds the
    scale factors of its own A rows and of all B rows of the tile, filled by
    four scale-factor warps): ragged M = 300 (the second CTA's rows partly
    past M) within tolerance of the oracle; M = 1100, N = 2048 with several
    tiles per pair, scale-factor slots and both accumulators reused, on
    sampled outputs; split 2 against the one-SM kernel's split 2 (the same K
    blocks per split and the same reduction)."""
    fmt = lq.BLOCK_FP8_UE8M0
    prob = make_problem(fmt, 300, 1024, 1280, seed=490)
    A, sa, B, sb = prob.device()
    vp = lq.make_variant(swap_ab=0, tile_n=128, persistent=2)
    C0 = lq.scaled_mm(fmt, A, sa, B, sb, variant=vp).clone()
    C1 = lq.scaled_mm(fmt, A, sa, B, sb, variant=vp)
    C2 = lq.scaled_mm(fmt, A, sa, B, sb, variant=lq.make_variant(swap_ab=0, tile_n=128, split_k=2, reduce=0,
                                                                   persistent=2))
    Cs = lq.scaled_mm(fmt, A, sa, B, sb, variant=lq.make_variant(swap_ab=0, tile_n=128, split_k=2, reduce=0))
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert torch.equal(C0, C1)
    assert_close(C0, prob.reference(), "ue8m0 pair")
    assert torch.equal(C2, Cs)
    assert_close(C2, prob.reference(), "ue8m0 pair split 2")
    big = make_problem(fmt, 1100, 2048, 1024, seed=491, outliers=False)
    A, sa, B, sb = big.device()
    Cb = lq.scaled_mm(fmt, A, sa, B, sb, variant=vp)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    rows = np.array([0, 127, 128, 255, 256, 700, 1023, 1024, 1099])
    cols = np.array([0, 7, 127, 128, 1023, 2047])
    ok, worst = O.within_tolerance(Cb.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)],
                                   big.reference(rows, cols))
    assert ok, worst


@pytest.mark.parametrize("S", [3, 12])
def test_ue8m0_pair_split_counts_bias_and_graph(cuda_device, S):
    """Split 3, and split 12 over T = 10 K blocks (empty splits); bias with
    and without Split-K; a graph replay gives the same bits."""
    fmt = lq.BLOCK_FP8_UE8M0
    prob = make_problem(fmt, 300, 1024, 1280, seed=495 + S)
    A, sa, B, sb = prob.device()
    v1 = lq.make_variant(swap_ab=0, tile_n=128, persistent=2)
    vs = lq.make_variant(swap_ab=0, tile_n=128, split_k=S, reduce=0, persistent=2)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, 300, 1024, 1280, vs))
    C = lq.scaled_mm(fmt, A, sa, B, sb, variant=vs)
    g = torch.Generator().manual_seed(496)
    bias = (torch.randn(1024, generator=g) * 0.5).to(torch.bfloat16).cuda()
    Cb1 = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=v1)
    Cbs = lq.scaled_mm_bias(fmt, A, sa, B, sb, bias, variant=vs)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    assert_close(C, prob.reference(), f"ue8m0 pair split {S}")
    refb = prob.reference() + bias.double().cpu().numpy()[None, :]
    assert_close(Cb1, refb, "ue8m0 pair bias")
    assert_close(Cbs, refb, f"ue8m0 pair split {S} bias")
    out = torch.empty_like(C)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(gr, stream=s):
            lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=vs, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        out.zero_()
        gr.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C)
    del gr
    assert lq.device_status(0) == 0


# --------------------------------------------------------------- stream-K (persistent = 3)
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("tn", [128, 256])
@pytest.mark.parametrize("M,N,K", [(300, 1000, 1040),      # fewer iterations than SMs: one K block per CTA
                                   (256, 1024, 25600)])    # 8 or 16 tiles of 200 K blocks over 148 CTAs
def test_streamk(cuda_device, fmt, tn, M, N, K):
    """Every tile finished by the CTA holding its last K block after adding
    the partials of up to ~20 earlier CTAs: within tolerance of the oracle
    (sampled at the deep size), INT8 accumulators exact, bitwise
    reproducible, also under graph replay (the ready flags return to zero)."""
    prob = make_problem(fmt, M, N, K, seed=421 + tn + M, outliers=False)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=0, tile_n=tn, persistent=3)
    lq.reserve_workspace(0, lq.workspace_bytes(fmt, M, N, K, v))
    if fmt == lq.W8A8_INT8:
        C0, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=v)
    else:
        C0 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v)
    C0 = C0.clone()
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    if K > 4096:
        rows = np.array([0, 1, 127, 128, 200, 255])
        cols = np.array([0, 5, 255, 256, 511, 512, 1000, 1023])
    else:
        rows, cols = np.arange(M), np.arange(N)
    name = {lq.FP8_DYNAMIC: O.FMT_FP8_DYNAMIC, lq.W8A8_INT8: O.FMT_W8A8_INT8}[fmt]
    ref = O.scaled_mm_ref(name, prob.qa[rows], prob.sa[rows], prob.qb[cols], prob.sb[cols])
    ok, worst = O.within_tolerance(C0.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)], ref)
    assert ok, worst
    if fmt == lq.W8A8_INT8:
        exact = O.acc_exact(O.FMT_W8A8_INT8, prob.qa[rows], prob.qb[cols])
        assert np.array_equal(acc.cpu().numpy().astype(np.int64)[np.ix_(rows, cols)], exact)
    out = torch.empty_like(C0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=v, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, C0)
    del g
    assert lq.device_status(0) == 0


def test_streamk_bias(cuda_device):
    prob = make_problem(lq.FP8_DYNAMIC, 256, 512, 8192, seed=431)
    A, sa, B, sb = prob.device()
    g = torch.Generator().manual_seed(432)
    bias = (torch.randn(512, generator=g) * 0.5).to(torch.bfloat16).cuda()
    v = lq.make_variant(swap_ab=0, tile_n=256, persistent=3)
    lq.reserve_workspace(0, lq.workspace_bytes("fp8_dynamic", 256, 512, 8192, v))
    C = lq.scaled_mm_bias(lq.FP8_DYNAMIC, A, sa, B, sb, bias, variant=v)
    torch.cuda.synchronize()
    assert_close(C, prob.reference() + bias.double().cpu().numpy()[None, :], "stream-K bias")
