"""The N-sliced (column-parallel) quantized linear: slice bounds and scale
slicing on one process, and on two gloo ranks on CPU the gathered output of
the slices equals the full layer's (the per-slice GEMM is injected: a CPU
product from the oracle, since these ranks have no GPU)."""

import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from quantized_linear_gemm_b200 import parallel  # noqa: E402


def test_shard_bounds():
    assert parallel.shard_bounds(4096, 4, 0, 8) == (0, 1024)
    assert parallel.shard_bounds(4096, 4, 3, 8) == (3072, 4096)
    assert parallel.shard_bounds(24576, 8, 5, 128) == (15360, 18432)
    with pytest.raises(ValueError):
        parallel.shard_bounds(4096, 3, 0, 8)         # 4096 / 3 is not a multiple of 8
    with pytest.raises(ValueError):
        parallel.shard_bounds(384, 2, 0, 128)        # 192-channel slices break 128-channel weight blocks
    with pytest.raises(ValueError):
        parallel.shard_bounds(4096, 2, 2, 8)


def test_slices_cover_the_layer_once():
    for N, world, align in [(6144, 8, 8), (51200, 4, 128), (4096, 1, 8)]:
        edges = [parallel.shard_bounds(N, world, r, align) for r in range(world)]
        assert edges[0][0] == 0 and edges[-1][1] == N
        assert all(a[1] == b[0] for a, b in zip(edges, edges[1:]))


def _cpu_gemm(fmt, A, a_s, B, b_s, stream=None):
    from oracle import lq_oracle as O
    if fmt == "block_fp8":
        C = O.blockwise_ref(A.numpy(), a_s.numpy(), B.numpy(), b_s.numpy())
    else:
        C = O.scaled_mm_ref(fmt, A.numpy(), a_s.numpy(), B.numpy(), b_s.numpy())
    return torch.from_numpy(C).to(torch.bfloat16)


def _cpu_gemm_bias(fmt, A, a_s, B, b_s, bias, stream=None):
    from oracle import lq_oracle as O
    C = O.scaled_mm_ref(fmt, A.numpy(), a_s.numpy(), B.numpy(), b_s.numpy())
    return torch.from_numpy(C + bias.double().numpy()[None, :]).to(torch.bfloat16)


def _problem(fmt, M, N, K, seed):
    from oracle import lq_oracle as O
    from quantized_linear_gemm_b200 import inputs
    x = inputs.activations(M, K, seed=seed).float().numpy()
    w = inputs.weights(N, K, seed=seed + 1).float().numpy()
    if fmt == "block_fp8":
        a, sa = O.quant_per_token_group128(x)
        b, sb = O.quant_weight_block128(w)
    else:
        a, sa = O.quant_per_token(x, fmt)
        b, sb = O.quant_per_channel(w, fmt)
    bias = torch.from_numpy(np.random.default_rng(seed).standard_normal(N)).to(torch.bfloat16)
    return [torch.from_numpy(np.ascontiguousarray(t)) for t in (a, sa, b, sb)] + [bias]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = []
        for fmt, N, with_bias in [("fp8_dynamic", 512, False), ("w8a8_int8", 256, True), ("block_fp8", 512, False)]:
            A, sa, B, sb, bias = _problem(fmt, 5, N, 256, seed=N)
            layer = parallel.ColumnParallelLinear.from_full(fmt, B, sb, bias if with_bias else None, rank, world)
            C = layer.forward(A, sa, gemm=_cpu_gemm, gemm_bias=_cpu_gemm_bias)
            full = (_cpu_gemm_bias(fmt, A, sa, B, sb, bias) if with_bias else _cpu_gemm(fmt, A, sa, B, sb))
            out.append(bool(torch.equal(C, full)) and tuple(C.shape) == (5, N))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_column_parallel_gather_equals_full_layer_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ok in res:
        assert all(ok), (rank, ok)
