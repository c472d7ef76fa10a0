"""Measure the dense 8-bit tensor-core peaks of this GPU with library GEMMs.

    python -m quantized_linear_gemm_b200.peaks [--out FILE] [--n 8192] [--seconds 4]

The roofline of the compute-bound (prefill) calls needs the dense e4m3 and
int8 tensor-core throughput of the GPU at hand.  This module measures them
the way the bf16 figure of the roofline was measured: an N x N x N GEMM of a
vendor library (torch._scaled_mm for e4m3 x e4m3 -> bf16 with per-tensor
scales, torch._int_mm for int8 x int8 -> int32), 2 N^3 operations per call,
timed with CUDA events as the best of 10 single calls ("burst", for a kernel
timed alone) and as the mean over back-to-back calls for a few seconds
("sustained", for a kernel timed inside a long step, under the power cap).
These library calls are a measuring stick only; they are not on the path.
"""

from __future__ import annotations

import argparse
import json
import time

import torch


def _time_one(fn) -> float:
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    fn()
    e.record()
    e.synchronize()
    return s.elapsed_time(e) * 1e-3


def _measure(fn, flops: float, seconds: float) -> dict:
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    burst = min(_time_one(fn) for _ in range(10))
    # sustained: batches of back-to-back calls until `seconds` have passed
    n, total = 0, 0.0
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(20):
            fn()
        e.record()
        e.synchronize()
        total += s.elapsed_time(e) * 1e-3
        n += 20
    return {"tflops_burst": round(flops / burst / 1e12, 1), "tflops_sustained": round(flops * n / total / 1e12, 1),
            "calls_sustained": n}


def measure(n: int = 8192, seconds: float = 4.0) -> dict:
    dev = torch.device("cuda")
    flops = 2.0 * n ** 3
    out = {"gpu_name": torch.cuda.get_device_name(dev), "n": n, "flops_per_call": flops,
           "how": "best of 10 single calls (burst) and back-to-back calls for "
                  f"{seconds:g} s (sustained), CUDA events, 2 N^3 operations per call"}
    g = torch.Generator(device=dev).manual_seed(0)
    a = (torch.randn(n, n, device=dev, generator=g) * 0.5).to(torch.float8_e4m3fn)
    b = (torch.randn(n, n, device=dev, generator=g) * 0.5).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev, dtype=torch.float32)
    try:
        out["e4m3"] = {"call": "torch._scaled_mm(A [N,K] row-major, B^T [K,N] column-major, per-tensor scales, "
                               "out_dtype=bf16)",
                       **_measure(lambda: torch._scaled_mm(a, b.t(), one, one, out_dtype=torch.bfloat16), flops,
                                  seconds)}
    except Exception as exc:   # a library without this kernel: say so, measure the rest
        out["e4m3"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    del a, b
    ai = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g)
    bi = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g)
    try:
        out["int8"] = {"call": "torch._int_mm(A [N,K] row-major, B^T [K,N] column-major) -> int32",
                       **_measure(lambda: torch._int_mm(ai, bi.t()), flops, seconds)}
    except Exception as exc:
        out["int8"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    return out


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--out", default=None, help="also write the JSON here")
    ap.add_argument("--n", type=int, default=8192)
    ap.add_argument("--seconds", type=float, default=4.0)
    a = ap.parse_args()
    res = measure(a.n, a.seconds)
    res["when"] = time.strftime("%Y-%m-%dT%H:%M:%SZ", time.gmtime())
    text = json.dumps(res, indent=1)
    print(text)
    if a.out:
        with open(a.out, "w") as f:
            f.write(text + "\n")


if __name__ == "__main__":
    main()
