"""GPU parity of scaled_mm (all formats, all variants) against the oracle,
through the C ABI.  bf16 outputs within |C - C_ref| <= 2^-7 |C_ref| +
1e-3 rms(C_ref); INT8 accumulators bit-exact."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import assert_close, make_problem

pytestmark = pytest.mark.gpu

FMTS = [lq.FP8_DYNAMIC, lq.W8A8_INT8, lq.BLOCK_FP8]
FMT_IDS = ["fp8", "int8", "block"]

# Every (orientation, tile) pair the library instantiates, with splits, both
# reduction modes and shallow / deep rings.
VARIANTS = []
for tn in (64, 128, 256):
    VARIANTS.append(dict(swap_ab=0, tile_n=tn, split_k=1, stages=2))
    VARIANTS.append(dict(swap_ab=0, tile_n=tn, split_k=4, stages=0, reduce=1))
for tn in (16, 32, 64):
    VARIANTS.append(dict(swap_ab=1, tile_n=tn, split_k=1, stages=3))
    VARIANTS.append(dict(swap_ab=1, tile_n=tn, split_k=2, stages=2, reduce=0))
    VARIANTS.append(dict(swap_ab=1, tile_n=tn, split_k=8, stages=4, reduce=1))
VARIANTS.append(dict(swap_ab=1, tile_n=32, split_k=16, stages=0, reduce=1, pdl=0))
for tn in (16, 32, 64):
    VARIANTS.append(dict(swap_ab=1, tile_n=tn, split_k=4, stages=2, reduce=2))
VARIANTS.append(dict(swap_ab=1, tile_n=16, split_k=16, stages=2, reduce=2, pdl=2))
for tn in (64, 128, 256):
    VARIANTS.append(dict(swap_ab=0, tile_n=tn, split_k=2, stages=0, reduce=2))
VARIANTS.append(dict(swap_ab=0, tile_n=64, split_k=16, stages=3, reduce=2))
VARIANTS.append(dict(swap_ab=0, tile_n=128, split_k=16, stages=4, reduce=0, pdl=0))


def _vid(v):
    return "{}{}-s{}-st{}-r{}".format("swap" if v["swap_ab"] else "std", v["tile_n"], v["split_k"],
                                      v.get("stages", 0), v.get("reduce", 1))


def _run(prob, variant=None, dev="cuda"):
    A, sa, B, sb = prob.device(dev)
    C = lq.scaled_mm(prob.fmt, A, sa, B, sb, variant=variant)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    return C


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("v", VARIANTS, ids=_vid)
def test_variants_small(cuda_device, fmt, v):
    """Ragged in every dimension: M = 37 (tile tails), N = 384 (a partial 256
    tile), K = 1152 (9 K tiles, uneven splits)."""
    if fmt == lq.BLOCK_FP8 and not v["swap_ab"] and v["tile_n"] == 256:
        pytest.skip("Block_FP8 Standard tiles stop at 128")
    prob = make_problem(fmt, 37, 384, 1152, seed=1)
    C = _run(prob, lq.make_variant(**v))
    assert_close(C, prob.reference(), _vid(v))


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8], ids=["fp8", "int8"])
@pytest.mark.parametrize("swap", [0, 1])
def test_ragged_k_tail(cuda_device, fmt, swap):
    """K = 1040: the last 128-wide K tile is 16 wide; TMA zero-fills the rest."""
    prob = make_problem(fmt, 5, 136, 1040, seed=2)
    v = lq.make_variant(swap_ab=swap, tile_n=16 if swap else 64, split_k=4, stages=2)
    assert_close(_run(prob, v), prob.reference(), "ragged K")


@pytest.mark.parametrize("v", VARIANTS, ids=_vid)
def test_int8_accumulator_bitexact(cuda_device, v):
    prob = make_problem(lq.W8A8_INT8, 37, 384, 1152, seed=3)
    A, sa, B, sb = prob.device()
    C, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=lq.make_variant(**v))
    torch.cuda.synchronize()
    ref = O.acc_exact(O.FMT_W8A8_INT8, prob.qa, prob.qb)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)
    assert_close(C, prob.reference(), "int8 C")


@pytest.mark.parametrize("S", [32, 64, 256])
def test_split_k_with_empty_splits(cuda_device, S):
    """K = 5120 -> 40 K tiles: S = 64 and 256 leave splits without work."""
    for fmt in FMTS:
        prob = make_problem(fmt, 3, 256, 5120, seed=4)
        for reduce in (0, 1):
            v = lq.make_variant(swap_ab=1, tile_n=16, split_k=S, stages=2, reduce=reduce)
            assert_close(_run(prob, v), prob.reference(), f"S={S} reduce={reduce} fmt={fmt}")


@pytest.mark.parametrize("fmt", [lq.FP8_DYNAMIC, lq.W8A8_INT8, lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0],
                         ids=["fp8", "int8", "block", "ue8m0"])
@pytest.mark.parametrize("swap,tn", [(1, 16), (1, 32), (0, 128)])
def test_split_counts_not_powers_of_two(cuda_device, fmt, swap, tn):
    """Split counts 3, 5, 7 and 12 (K = 2304: 18 K tiles, splits of one to
    six tiles) with the separate reduction and with the last arriver: the
    same partials summed in the same order, so identical bits; within
    tolerance of the oracle; W8A8_INT8 accumulators exact."""
    M, N, K = (40, 512, 2304) if swap else (200, 512, 2304)
    prob = make_problem(fmt, M, N, K, seed=16 + tn)
    A, sa, B, sb = prob.device()
    ref = prob.reference()
    for S in (3, 5, 7, 12):
        outs = []
        for red in (0, 1):
            v = lq.make_variant(swap_ab=swap, tile_n=tn, split_k=S, stages=2, reduce=red)
            lq.reserve_workspace(0, lq.workspace_bytes(fmt, M, N, K, v))
            outs.append(lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone())
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]), f"S={S}"
        assert_close(outs[0], ref, f"S={S}")
        if fmt == lq.W8A8_INT8:
            _, acc = lq.scaled_mm_i32acc(A, sa, B, sb, variant=v)
            torch.cuda.synchronize()
            assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.acc_exact(O.FMT_W8A8_INT8, prob.qa, prob.qb))
    assert lq.device_status(0) == 0


def test_config0_fp8_standard(cuda_device):
    """FP8_Dynamic, M = 16, N = K = 2048, A ~ N(0,1), B ~ N(0,0.02), Standard."""
    x = inputs.activations(16, 2048, seed=0, outliers=False).float().numpy()
    w = inputs.weights(2048, 2048, seed=0).float().numpy()
    qa, sa = O.quant_per_token(x, O.FMT_FP8_DYNAMIC)
    qb, sb = O.quant_per_channel(w, O.FMT_FP8_DYNAMIC)
    ref = O.scaled_mm_ref(O.FMT_FP8_DYNAMIC, qa, sa, qb, sb)
    A = torch.from_numpy(qa).cuda()
    B = torch.from_numpy(qb).cuda()
    for tn in (64, 128, 256):
        C = lq.scaled_mm(lq.FP8_DYNAMIC, A, torch.from_numpy(sa).cuda(), B, torch.from_numpy(sb).cuda(),
                         variant=lq.make_variant(swap_ab=0, tile_n=tn, split_k=1))
        assert_close(C, ref, f"config 0 tile {tn}")


def test_quant_then_gemm_end_to_end(cuda_device):
    """bf16 activations quantized on the GPU, then scaled_mm: equals the oracle on the same bf16."""
    x = inputs.activations(8, 4096, seed=9)
    w = inputs.weights(512, 4096, seed=10)
    for fmt in ("fp8_dynamic", "w8a8_int8"):
        qb, sb = lq.quant_per_token(fmt, w.cuda())
        qa, sa = lq.quant_per_token(fmt, x.cuda())
        C = lq.scaled_mm(fmt, qa, sa, qb, sb)
        ra, rsa = O.quant_per_token(x.float().numpy(), fmt)
        rb, rsb = O.quant_per_channel(w.float().numpy(), fmt)
        assert_close(C, O.scaled_mm_ref(fmt, ra, rsa, rb, rsb), fmt)
    qb, sb = lq.quant_weight_block128(w.cuda())
    qa, sa = lq.quant_per_token_group128(x.cuda())
    C = lq.scaled_mm("block_fp8", qa, sa, qb, sb)
    ra, rsa = O.quant_per_token_group128(x.float().numpy())
    rb, rsb = O.quant_weight_block128(w.float().numpy())
    assert_close(C, O.blockwise_ref(ra, rsa, rb, rsb), "block")


def test_degenerate_sizes(cuda_device):
    dev = cuda_device
    # K = 0: C = 0
    A = torch.empty((4, 0), dtype=torch.uint8, device=dev)
    B = torch.empty((16, 0), dtype=torch.uint8, device=dev)
    C = torch.full((4, 16), 7.0, dtype=torch.bfloat16, device=dev)
    lq.scaled_mm(lq.FP8_DYNAMIC, A, torch.ones(4, device=dev), B, torch.ones(16, device=dev), C=C)
    assert torch.all(C == 0)
    # M = 0: no-op
    A = torch.empty((0, 128), dtype=torch.uint8, device=dev)
    B = torch.zeros((16, 128), dtype=torch.uint8, device=dev)
    C = lq.scaled_mm(lq.FP8_DYNAMIC, A, torch.ones(0, device=dev), B, torch.ones(16, device=dev))
    assert C.shape == (0, 16)
    # smallest legal N (8) and K (16), single token
    prob = make_problem(lq.FP8_DYNAMIC, 1, 8, 16, seed=11)
    for v in (lq.make_variant(swap_ab=1, tile_n=16), lq.make_variant(swap_ab=0, tile_n=64)):
        assert_close(_run(prob, v), prob.reference(), "tiny")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
def test_scale_linearity_bitexact(cuda_device, fmt):
    """Doubling a_s of one token doubles that row of C exactly (x2 commutes with
    fp32 arithmetic and bf16 rounding) and leaves the others unchanged."""
    prob = make_problem(fmt, 8, 256, 1024, seed=12)
    A, sa, B, sb = prob.device()
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=4)
    C1 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone()
    sa2 = sa.clone()
    sa2[3] *= 2
    C2 = lq.scaled_mm(fmt, A, sa2, B, sb, variant=v)
    torch.cuda.synchronize()
    assert torch.equal(C2[3].float(), 2 * C1[3].float())
    keep = [0, 1, 2, 4, 5, 6, 7]
    assert torch.equal(C2[keep], C1[keep])


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
def test_deterministic_and_graph_replay(cuda_device, fmt):
    """Each variant is bitwise reproducible, eager and under CUDA-graph replay."""
    prob = make_problem(fmt, 16, 512, 2048, seed=13)
    A, sa, B, sb = prob.device()
    lq.init_device(0)
    for v in (lq.make_variant(swap_ab=1, tile_n=16, split_k=8, reduce=1),
              lq.make_variant(swap_ab=1, tile_n=16, split_k=8, reduce=0),
              lq.make_variant(swap_ab=0, tile_n=128, split_k=2)):
        lq.reserve_workspace(0, lq.workspace_bytes(fmt, 16, 512, 2048, v))
        C0 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone()
        C1 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone()
        assert torch.equal(C0, C1)
        out = torch.empty_like(C0)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for _ in range(3):
                    lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=v, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        for _ in range(3):
            out.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, C0)
        del g
        assert_close(C0, prob.reference(), "graph")
    assert lq.device_status(0) == 0


def _random_operands(fmt, M, N, K, seed):
    """Random finite codes and positive scales, generated on the device (a
    run-to-run invariant needs no reference values)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)

    def codes(rows):
        if fmt == lq.W8A8_INT8:
            return torch.randint(-127, 128, (rows, K), generator=g, device="cuda", dtype=torch.int8)
        q = torch.randint(0, 256, (rows, K), generator=g, device="cuda", dtype=torch.uint8)
        return torch.where((q & 0x7F) == 0x7F, torch.zeros_like(q), q)   # no NaN codes

    def scales(shape):
        return torch.rand(shape, generator=g, device="cuda") * 1e-3 + 1e-5

    block = fmt == lq.BLOCK_FP8
    A, B = codes(M), codes(N)
    sa = scales((M, K // 128) if block else (M,))
    sb = scales((N // 128, K // 128) if block else (N,))
    return A, sa, B, sb


DEEP_K = [  # (M, N, K, variant): Qwen3-32B down (K = 25600, 200 K tiles) in prefill and decode tiles
    (2048, 1024, 25600, dict(swap_ab=0, tile_n=128, split_k=1, stages=4, reduce=2, pdl=2)),
    (2048, 1024, 25600, dict(swap_ab=0, tile_n=64, split_k=1, stages=3, reduce=2, pdl=2)),
    (256, 1024, 25600, dict(swap_ab=0, tile_n=128, split_k=4, stages=3, reduce=2, pdl=2)),
    (8, 5120, 25600, dict(swap_ab=1, tile_n=16, split_k=8, stages=4, reduce=2, pdl=2)),
    (8, 5120, 25600, dict(swap_ab=1, tile_n=16, split_k=8, stages=4, reduce=0, pdl=2)),
    (8, 5120, 25600, None),
]


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("M,N,K,vd", DEEP_K, ids=lambda x: None if not isinstance(x, (dict, type(None))) else
                         ("table" if x is None else _vid(x)))
def test_deep_k_bitwise_reproducible(cuda_device, fmt, M, N, K, vd):
    """Run to run the same bits at the deepest K of the workloads: every
    variant sums its partial products and its splits in one fixed order, so
    repeated calls (eager, back to back on one stream) must agree bit for bit;
    and sampled outputs within tolerance of the oracle."""
    A, sa, B, sb = _random_operands(fmt, M, N, K, seed=M + N)
    v = None if vd is None else lq.make_variant(**vd)
    if v is not None:
        lq.reserve_workspace(0, lq.workspace_bytes(fmt, M, N, K, v))
    C0 = lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone()
    out = torch.empty_like(C0)
    for _ in range(3):
        out.zero_()
        lq.scaled_mm(fmt, A, sa, B, sb, C=out, variant=v)
        torch.cuda.synchronize()
        assert torch.equal(out, C0)
    assert torch.isfinite(C0.float()).all()
    # and the oracle on sampled outputs (exact products of the random codes)
    qa, qb = A.cpu().numpy(), B.cpu().numpy()
    san, sbn = sa.cpu().numpy().astype(np.float64), sb.cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(M + N + K)
    rows = np.sort(rng.choice(M, size=min(M, 6), replace=False))
    cols = np.sort(rng.choice(N, size=12, replace=False))
    if fmt == lq.BLOCK_FP8:
        ref = np.stack([O.blockwise_ref(qa[rows], san[rows], qb[n:n + 1], sbn[n // 128:n // 128 + 1])[:, 0]
                        for n in cols], axis=1)
    else:
        name = O.FMT_FP8_DYNAMIC if fmt == lq.FP8_DYNAMIC else O.FMT_W8A8_INT8
        ref = O.scaled_mm_ref(name, qa[rows], san[rows], qb[cols], sbn[cols])
    got = C0.float().cpu().numpy().astype(np.float64)[np.ix_(rows, cols)]
    ok, worst = O.within_tolerance(got, ref)
    assert ok, worst
    assert lq.device_status(0) == 0


def test_default_variant_selection_runs(cuda_device):
    """variant = NULL takes the table / heuristic choice."""
    for fmt in FMTS:
        for M in (1, 24, 100):
            prob = make_problem(fmt, M, 256, 1024, seed=14)
            assert_close(_run(prob, None), prob.reference(), f"default fmt={fmt} M={M}")


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("swap,tn", [(1, 16), (1, 32), (1, 64), (0, 64), (0, 128), (0, 256)])
def test_reduce_modes_bitwise_identical(cuda_device, fmt, swap, tn):
    """Separate kernel, last arriver and cluster reduction sum the same
    partials in the same order: identical bits, and within tolerance."""
    if fmt == lq.BLOCK_FP8 and not swap and tn == 256:
        pytest.skip("Block_FP8 Standard tiles stop at 128")
    prob = make_problem(fmt, 40, 512, 2304, seed=15)
    A, sa, B, sb = prob.device()
    ref = prob.reference()
    for S in (2, 4, 8, 16):
        outs = []
        for red in (0, 1, 2):
            v = lq.make_variant(swap_ab=swap, tile_n=tn, split_k=S, stages=2, reduce=red)
            outs.append(lq.scaled_mm(fmt, A, sa, B, sb, variant=v).clone())
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2]), f"S={S}"
        assert_close(outs[2], ref, f"cluster S={S}")
    assert lq.device_status(0) == 0
