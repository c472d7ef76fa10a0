"""GPU parity of the grouped (mixture-of-experts) quantized GEMM, called
through the C ABI: C within the suite's tolerance of the oracle, and bit for
bit the rows that a dense lq_scaled_mm per expert gives with the same
variant; empty experts, one crowded expert, a single expert, malformed
offset tables (clamped by the kernel) and the Qwen3-30B-A3B expert shapes."""

import numpy as np
import pytest
import torch

from oracle import lq_oracle as O
from oracle import moe_oracle as MO
from quantized_linear_gemm_b200 import inputs, lq

from _lqtest import bf16_to_f64

pytestmark = pytest.mark.gpu


def _problem(fmt, counts, N, K, seed):
    T, E = int(sum(counts)), len(counts)
    x = inputs.activations(max(T, 1), K, seed=seed).float().numpy()[:T]
    w = inputs.weights(E * N, K, seed=seed + 1).float().numpy().reshape(E, N, K)
    a, sa = O.quant_per_token(x, fmt)
    b = np.empty((E, N, K), dtype=np.int8 if fmt == "w8a8_int8" else np.uint8)
    sb = np.empty((E, N), dtype=np.float32)
    for e in range(E):
        b[e], sb[e] = O.quant_per_channel(w[e], fmt)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return a, sa, b, sb, off


def _dev(*arrays):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrays]


def _run(fmt, a, sa, b, sb, off, variant=None):
    A, SA, B, SB, OFF = _dev(a, sa, b, sb, off)
    C = lq.grouped_scaled_mm(fmt, A, SA, B, SB, OFF, variant=variant)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    return C


def _check(fmt, C, a, sa, b, sb, off, variant):
    ref = MO.grouped_scaled_mm_ref(fmt, a, sa, b, sb, off)
    ok, worst = O.within_tolerance(bf16_to_f64(C), ref)
    assert ok, worst
    if variant is None:   # the grouped heuristic and the dense table may pick different variants
        return
    # each expert's rows equal a dense call with the same variant, bit for bit
    A, SA, B, SB = _dev(a, sa, b, sb)
    for e in range(b.shape[0]):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            Ce = lq.scaled_mm(fmt, A[lo:hi].contiguous(), SA[lo:hi].contiguous(), B[e], SB[e], variant=variant)
            torch.cuda.synchronize()
            assert torch.equal(C[lo:hi], Ce), e


VARIANTS = [None, dict(swap_ab=1, tile_n=16, split_k=1, stages=4), dict(swap_ab=1, tile_n=16, split_k=4, stages=2),
            dict(swap_ab=1, tile_n=32, split_k=2, stages=3), dict(swap_ab=1, tile_n=64, split_k=8, stages=2)]


@pytest.mark.parametrize("fmt", ["fp8_dynamic", "w8a8_int8"])
@pytest.mark.parametrize("vd", VARIANTS, ids=lambda v: "table" if v is None else f"tn{v['tile_n']}-s{v['split_k']}")
def test_grouped_small_experts(cuda_device, fmt, vd):
    counts = [3, 0, 1, 17, 0, 0, 5, 40, 2, 1]   # empty experts, a crowded one, ragged tiles
    a, sa, b, sb, off = _problem(fmt, counts, 384, 1040, seed=1)   # ragged K (1040 = 8 x 128 + 16)
    v = None if vd is None else lq.make_variant(reduce=2, **vd)
    C = _run(fmt, a, sa, b, sb, off, v)
    _check(fmt, C, a, sa, b, sb, off, v)


@pytest.mark.parametrize("layer", ["gate_up", "down"])
@pytest.mark.parametrize("tokens", [1, 8, 64])
def test_grouped_qwen3_moe_decode(cuda_device, layer, tokens):
    K, N = inputs.QWEN3_30B_A3B_EXPERTS[layer]
    E, k = inputs.QWEN3_30B_A3B_NUM_EXPERTS, inputs.QWEN3_30B_A3B_TOP_K
    counts = inputs.expert_counts(tokens, E, k, seed=inputs.stable_seed("moe", layer, tokens))
    a, sa, b, sb, off = _problem("fp8_dynamic", counts, N, K, seed=tokens)
    C = _run("fp8_dynamic", a, sa, b, sb, off)
    ref = MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b, sb, off)
    ok, worst = O.within_tolerance(bf16_to_f64(C), ref)
    assert ok, worst


def test_single_expert_is_the_dense_call(cuda_device):
    a, sa, b, sb, off = _problem("fp8_dynamic", [37], 512, 2048, seed=5)
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=2, stages=4, reduce=2)
    C = _run("fp8_dynamic", a, sa, b, sb, off, v)
    A, SA, B, SB = _dev(a, sa, b, sb)
    assert torch.equal(C, lq.scaled_mm("fp8_dynamic", A, SA, B[0], SB[0], variant=v))


def test_malformed_offsets_stay_inside_C(cuda_device):
    """Offsets past T or decreasing: the kernel uses [H(e-1), H(e)) with H the
    running max of the clamped offsets; rows outside every expert are left
    as they were and nothing is written past C."""
    a, sa, b, sb, _ = _problem("fp8_dynamic", [20], 256, 512, seed=6)
    b3 = np.concatenate([b, b, b])
    sb3 = np.concatenate([sb, sb * 2, sb * 3])
    bad = np.array([0, 10, 5, 200], dtype=np.int32)           # H = 10, 10, 20
    A, SA, B, SB, OFF = _dev(a, sa, b3, sb3, bad)
    guard = torch.full((24, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    C = guard[:20]
    lq.grouped_scaled_mm("fp8_dynamic", A, SA, B, SB, OFF, C=C)
    torch.cuda.synchronize()
    assert lq.device_status(0) == 0
    ref = MO.grouped_scaled_mm_ref("fp8_dynamic", a, sa, b3, sb3, np.array([0, 10, 10, 20]))
    ok, worst = O.within_tolerance(bf16_to_f64(C), ref)
    assert ok, worst
    assert torch.all(guard[20:] == 7.0)


def test_grouped_is_deterministic_and_graph_replayable(cuda_device):
    counts = inputs.expert_counts(16, 64, 4, seed=7)
    a, sa, b, sb, off = _problem("w8a8_int8", counts, 256, 768, seed=7)
    A, SA, B, SB, OFF = _dev(a, sa, b, sb, off)
    v = lq.make_variant(swap_ab=1, tile_n=16, split_k=2, stages=3, reduce=2)
    C1 = lq.grouped_scaled_mm("w8a8_int8", A, SA, B, SB, OFF, variant=v)
    s = torch.cuda.Stream()
    C2 = torch.empty_like(C1)
    with torch.cuda.stream(s):
        lq.grouped_scaled_mm("w8a8_int8", A, SA, B, SB, OFF, C=C2, variant=v, stream=s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            lq.grouped_scaled_mm("w8a8_int8", A, SA, B, SB, OFF, C=C2, variant=v, stream=s)
    C2.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(C1, C2)
