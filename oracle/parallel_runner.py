"""Runs the oracle's exact products on every host core, for the CPU baseline.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs may import or run this module.  The library under
``quantized_linear_gemm_b200/`` never calls it, links it or shares code with it.

The oracle's accumulation (numpy int64 matmul) uses one core.  To time it on
all the host's cores, the output columns of each linear layer are split into
slices and the slices are computed by worker processes (started with
``spawn``, so that a process that already uses a GPU can start them).  Each
worker quantizes the layer's activations and computes the exact product of
its slice with the oracle's own functions, unchanged; the operands are
shared through memory-mapped .npy files written once by the parent.  Nothing
here changes what the oracle computes.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import tempfile
import time

import numpy as np

_DATA: dict = {}


def _init(paths: dict) -> None:
    for key, path in paths.items():
        _DATA[key] = np.load(path, mmap_mode="r")


def _product(task) -> float:
    """Quantize layer li's activations, then the exact product of weight rows
    [c0, c1); returns the seconds it took."""
    from oracle import lq_oracle as O
    from oracle import ue8m0_oracle as U

    fmt, li, c0, c1 = task
    x = np.asarray(_DATA[f"x{li}"])
    qb = np.asarray(_DATA[f"qb{li}"][c0:c1])
    sb_all = _DATA[f"sb{li}"]
    t0 = time.perf_counter()
    if fmt == "block_fp8_ue8m0":
        qa, sa = U.quant_per_token_group128_ue8m0(x)
        U.blockwise_ue8m0_ref(qa, sa, qb, np.asarray(sb_all[c0 // 128:c1 // 128]))
    elif fmt == "block_fp8":
        qa, sa = O.quant_per_token_group128(x)
        O.blockwise_ref(qa, sa, qb, np.asarray(sb_all[c0 // 128:c1 // 128]))
    else:
        qa, sa = O.quant_per_token(x, fmt)
        O.scaled_mm_ref(fmt, qa, sa, qb, np.asarray(sb_all[c0:c1]))
    return time.perf_counter() - t0


def time_all_cores(fmt: str, layers: list, budget_s: float, workers: int | None = None) -> dict:
    """layers: [(x [M, K] float64 bf16 values, qb [N, K] codes, sb scales)].
    Repeats one round (every layer, every column slice) until `budget_s` has
    passed; returns {"rounds", "seconds", "workers"} (wall time of the rounds)."""
    workers = workers or (os.cpu_count() or 1)
    with tempfile.TemporaryDirectory() as tmp:
        paths = {}
        tasks = []
        for li, (x, qb, sb) in enumerate(layers):
            for key, arr in ((f"x{li}", x), (f"qb{li}", qb), (f"sb{li}", sb)):
                paths[key] = os.path.join(tmp, key + ".npy")
                np.save(paths[key], np.ascontiguousarray(arr))
            N = qb.shape[0]
            step = 128 if fmt in ("block_fp8", "block_fp8_ue8m0") else 8
            per = max(step, -(-N // workers) // step * step)   # slices of whole weight blocks
            for c0 in range(0, N, per):
                tasks.append((fmt, li, c0, min(N, c0 + per)))
        ctx = mp.get_context("spawn")
        with ctx.Pool(processes=workers, initializer=_init, initargs=(paths,)) as pool:
            pool.map(_product, tasks[:workers], chunksize=1)   # workers started and warm
            rounds, t0 = 0, time.perf_counter()
            while True:
                pool.map(_product, tasks, chunksize=1)
                rounds += 1
                dt = time.perf_counter() - t0
                if dt > budget_s or rounds >= 50:
                    break
    return {"rounds": rounds, "seconds": dt, "workers": workers, "tasks_per_round": len(tasks)}
