#!/usr/bin/env python
"""Benchmark of the quantized linear-layer GEMM hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl lq|reference]

One step = one pass of the whole hot path over one batch: for every decode
size M in {1, 2, 4, 8, 16, 24, 32} and every linear of a Qwen3 layer, the
bf16 activations are quantized (lq_quant_per_token / _group128) and
multiplied with the pre-quantized weights (lq_scaled_mm, variant from the
dispatch table).  The step is captured once in a CUDA graph and replayed.
Weights are kept in several copies that are rotated between M points so
that every weight read comes from HBM (more than 2x the L2 capacity passes
between two reads of one copy).

The end-to-end figure (`e2e`) copies every step's bf16 activations from
pinned host memory to the device and every output back, inside the timed
region; two buffer sets and two copy streams overlap those copies with the
neighbouring steps' kernels.

The metric is HBM throughput of algorithmic bytes (weights + activations +
scales + outputs, plus the quantizers' reads and writes) per second; TFLOP/s
and the per-shape breakdown are reported beside it.  Multi-GPU runs are
replicas (each rank runs the whole step on its own GPU; no collective is
part of the hot path) and report the aggregate.
"""

from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from quantized_linear_gemm_b200 import inputs, lq  # noqa: E402

CONFIGS = {
    # name: (format, model shapes, M list)
    "qwen3-8b-fp8-decode": ("fp8_dynamic", inputs.QWEN3_8B, inputs.DECODE_M),
    "qwen3-8b-int8-decode": ("w8a8_int8", inputs.QWEN3_8B, inputs.DECODE_M),
    "qwen3-32b-block-decode": ("block_fp8", inputs.QWEN3_32B, inputs.DECODE_M),
    "qwen3-32b-fp8-prefill": ("fp8_dynamic", {k: inputs.QWEN3_32B[k] for k in ("gate_up", "down")}, inputs.PREFILL_M),
    "qwen3-32b-int8-prefill": ("w8a8_int8", {k: inputs.QWEN3_32B[k] for k in ("gate_up", "down")}, inputs.PREFILL_M),
    "qwen3-32b-block-prefill": ("block_fp8", {k: inputs.QWEN3_32B[k] for k in ("gate_up", "down")}, inputs.PREFILL_M),
    # Block_FP8 with power-of-two (UE8M0) scales: the tensor core's block-scaled MMA
    "qwen3-32b-ue8m0-decode": ("block_fp8_ue8m0", inputs.QWEN3_32B, inputs.DECODE_M),
    "qwen3-32b-ue8m0-prefill": ("block_fp8_ue8m0", {k: inputs.QWEN3_32B[k] for k in ("gate_up", "down")},
                                inputs.PREFILL_M),
}
BLOCK_FMTS = ("block_fp8", "block_fp8_ue8m0")
DEFAULT_CONFIG = "qwen3-8b-fp8-decode"
L2_BYTES = 126 * 2 ** 20


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def tensor_peak_8bit(fmt: str, peaks: dict) -> tuple[float, str]:
    """(TFLOP/s, source) of the dense 8-bit tensor-core peak for a kernel timed
    inside a long step: the sustained figure measured on this machine with a
    library GEMM (profiles/tensor_peaks_8bit.json, written by
    ``python -m quantized_linear_gemm_b200.peaks``), e4m3 for the FP8 formats
    and int8 for W8A8_INT8; without that file, twice the measured bf16
    sustained figure (the nominal 8-bit : bf16 ratio)."""
    p = os.path.join(ROOT, "profiles", "tensor_peaks_8bit.json")
    key = "int8" if fmt == "w8a8_int8" else "e4m3"
    if os.path.exists(p):
        d = json.load(open(p)).get(key, {})
        if "tflops_sustained" in d:
            return float(d["tflops_sustained"]), f"measured {key} sustained ({d.get('call', 'library GEMM')})"
    return 2.0 * peaks["bf16_tflops_sustained"], f"{peaks['source']} bf16 sustained x 2 (nominal 8-bit : bf16 ratio)"


def kernel_sources_digest() -> str:
    """First 16 hex of sha256 over the CUDA sources (without the dispatch table)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_linear_gemm_b200", "csrc")
    files = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh")) +
                   glob.glob(os.path.join(csrc, "*.h")))
    for f in files:
        if not f.endswith("dispatch_table.inc"):
            h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(config: str, kernel: str):
    """DRAM bytes per step of the step's `kernel` launches ("fused" or
    "scaled_mm") from the committed ncu summary, or None when there is none
    or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", f"traffic_{config.replace('-', '_')}_{kernel}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_sources_sha256_16") != kernel_sources_digest():
        return None
    return int(d["dram_bytes_per_step"])


# ------------------------------------------------------- multi-rank timing
def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms * 1e-3)


# ------------------------------------------------------------------ sizes
def gemm_bytes(fmt: str, M: int, N: int, K: int) -> int:
    return lq.Problem(lq.FORMATS[fmt], M, N, K).bytes


def quant_bytes(fmt: str, M: int, K: int) -> int:
    """bf16 read + codes written + scales written."""
    scales = {"block_fp8": 4 * M * (K // 128), "block_fp8_ue8m0": M * (K // 128)}.get(fmt, 4 * M)
    return 2 * M * K + M * K + scales


# -------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        exe = shutil.which("nvidia-smi")
        if not exe:
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.proc = subprocess.Popen([exe, "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                      "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 active=parts[4], hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded), "power_w_max": max(r["power"] for r in rows)}


# ------------------------------------------------------------ workload
class Workload:
    """Device buffers of one configuration: rotated weight copies, bf16
    activations, codes, scales and outputs of every (M, layer) call."""

    def __init__(self, config: str, device: torch.device, copies: int = 3, seed: int = 0, ms=None, layers=None):
        self.config = config
        self.fmt, self.layers, self.ms = CONFIGS[config]
        if ms:   # a subset of the configuration's token counts (profiling of one shape)
            self.ms = [m for m in self.ms if m in ms]
        if layers:
            self.layers = {k: v for k, v in self.layers.items() if k in layers}
        self.device = device
        self.copies = copies
        f = self.fmt
        self.weights = {}   # layer -> list of (codes, scales)
        for li, (layer, (K, N)) in enumerate(self.layers.items()):
            w = inputs.weights(N, K, seed=inputs.stable_seed(config, "W", layer, seed)).to(device)
            if f == "block_fp8":
                q, s = lq.quant_weight_block128(w)
            elif f == "block_fp8_ue8m0":
                q, s = lq.quant_weight_block128_ue8m0(w)
            else:
                q, s = lq.quant_per_token(f, w)
            # enough copies that more than 2x L2 is streamed between two reads of one copy
            n_copies = max(copies, -(-2 * L2_BYTES // (N * K)) + 1)
            reps = [(q, s)]
            for _ in range(n_copies - 1):
                reps.append((q.clone(), s.clone()))
            self.weights[layer] = reps
            del w
        # one flat bf16 buffer for every activation, one for every output
        self.calls = []
        x_off = c_off = 0
        for M in self.ms:
            for layer, (K, N) in self.layers.items():
                self.calls.append(dict(M=M, layer=layer, K=K, N=N, x_off=x_off, c_off=c_off))
                x_off += -(-M * K // 64) * 64
                c_off += -(-M * N // 64) * 64
        self.x_all = torch.empty(x_off, dtype=torch.bfloat16, device=device)
        self.c_all = torch.empty(c_off, dtype=torch.bfloat16, device=device)
        code_dt = torch.int8 if f == "w8a8_int8" else torch.uint8
        for i, c in enumerate(self.calls):
            M, K, N = c["M"], c["K"], c["N"]
            x = inputs.activations(M, K, seed=inputs.stable_seed(config, "A", c["layer"], M, seed))
            c["x"] = self.x_all[c["x_off"]:c["x_off"] + M * K].view(M, K)
            c["x"].copy_(x)
            c["C"] = self.c_all[c["c_off"]:c["c_off"] + M * N].view(M, N)
            c["q"] = torch.empty((M, K), dtype=code_dt, device=device)
            if f == "block_fp8_ue8m0":
                c["s"] = torch.empty((M, K // 128), dtype=torch.uint8, device=device)
            else:
                c["s"] = torch.empty((M, K // 128) if f == "block_fp8" else (M,), dtype=torch.float32, device=device)
            c["copy"] = self.ms.index(M) % len(self.weights[c["layer"]])
            c["variant"] = lq.select_variant(f, M, N, K)
        self.x_host = torch.empty(self.x_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.x_host.copy_(self.x_all)
        self.c_host = torch.empty(self.c_all.shape, dtype=torch.bfloat16, pin_memory=True)
        ws = max(lq.workspace_bytes(f, c["M"], c["N"], c["K"], c["variant"]) for c in self.calls)
        lq.reserve_workspace(device.index, ws)

    # bytes / flops of one step
    @property
    def gemm_bytes(self) -> int:
        return sum(gemm_bytes(self.fmt, c["M"], c["N"], c["K"]) for c in self.calls)

    @property
    def quant_bytes(self) -> int:
        return sum(quant_bytes(self.fmt, c["M"], c["K"]) for c in self.calls)

    @property
    def flops(self) -> int:
        return sum(2 * c["M"] * c["N"] * c["K"] for c in self.calls)

    def launches_per_step(self, gemm=True, quant=True, fused=False) -> int:
        n = 0
        for c in self.calls:
            if fused:
                v = c["variant"]
                fusable = v.swap_ab == 1 and v.split_k <= 16 and v.split_k * v.tile_n <= 512
                n += 1 if fusable else 2
                continue
            v = c["variant"]
            if quant:
                n += 1
            if gemm:
                n += 1 + (1 if (v.split_k > 1 and v.reduce == 0) else 0)
        return n

    def bind(self, x_all: torch.Tensor, c_all: torch.Tensor) -> None:
        """Point every call's activations / outputs into the given flat buffers."""
        for c in self.calls:
            M, K, N = c["M"], c["K"], c["N"]
            c["x"] = x_all[c["x_off"]:c["x_off"] + M * K].view(M, K)
            c["C"] = c_all[c["c_off"]:c["c_off"] + M * N].view(M, N)

    def quant(self, c, stream):
        if self.fmt == "block_fp8":
            lq.quant_per_token_group128(c["x"], c["q"], c["s"], stream=stream)
        elif self.fmt == "block_fp8_ue8m0":
            lq.quant_per_token_group128_ue8m0(c["x"], c["q"], c["s"], stream=stream)
        else:
            lq.quant_per_token(self.fmt, c["x"], c["q"], c["s"], stream=stream)

    def gemm(self, c, stream, copy=None, variant=None):
        reps = self.weights[c["layer"]]
        qb, sb = reps[c["copy"] if copy is None else copy % len(reps)]
        lq.scaled_mm(self.fmt, c["q"], c["s"], qb, sb, C=c["C"], variant=variant or c["variant"], stream=stream)

    def fused(self, c, stream):
        qb, sb = self.weights[c["layer"]][c["copy"]]
        lq.quant_scaled_mm(self.fmt, c["x"], qb, sb, C=c["C"], q=c["q"], s=c["s"], variant=c["variant"],
                           stream=stream)

    def step(self, stream, gemm=True, quant=True, fused=False):
        for c in self.calls:
            if fused:
                self.fused(c, stream)
                continue
            if quant:
                self.quant(c, stream)
            if gemm:
                self.gemm(c, stream)


def producer_bytes(op: str, M: int, K: int, residual: bool) -> int:
    """Algorithmic HBM bytes of one producer-side fused quantizer call: bf16
    inputs read once, codes and fp32 scales written once (plus the residual
    read and written back, and the RMSNorm gain)."""
    per_block = op.endswith("per_block_quant")
    scales = 4 * M * (K // 128) if per_block else 4 * M
    if op.startswith("rms_norm"):
        return 2 * M * K + (4 * M * K if residual else 0) + 2 * K + M * K + scales
    return 4 * M * K + M * K + scales


def producer_measurements(peaks, stream) -> list:
    """Per-call time of the four producer-side fused quantizers at the
    Qwen3-8B sizes (hidden 4096 for RMSNorm, intermediate 12288 for
    SiLU-and-mul): decode rows (M = 8, 32) and a prefill batch (M = 4096),
    graph-replayed, with enough input copies that more than 2 x L2 streams
    between two reads of one copy."""
    out = []
    l2 = 126 * 2 ** 20
    K, I = 4096, 12288
    w = torch.ones(K, dtype=torch.bfloat16, device="cuda")
    for M in (8, 32, 4096):
        for op in ("rms_norm_dynamic_per_token_quant", "rms_norm_per_block_quant",
                   "silu_and_mul_dynamic_per_token_quant", "silu_and_mul_per_block_quant"):
            rms = op.startswith("rms_norm")
            cols = K if rms else I
            in_bytes = M * (K * 4 if rms else 2 * I * 2)
            copies = max(2, 2 * l2 // in_bytes + 1) if M >= 1024 else 2
            xs = [inputs.activations(M, 2 * cols if not rms else cols, seed=inputs.stable_seed(op, M, r)).cuda()
                  for r in range(copies)]
            rs = [inputs.activations(M, cols, seed=inputs.stable_seed(op, "res", M, r)).cuda()
                  for r in range(copies)] if rms else None
            q = torch.empty((M, cols), dtype=torch.uint8, device="cuda")
            per_block = op.endswith("per_block_quant")
            sc = torch.empty((M, cols // 128) if per_block else (M,), dtype=torch.float32, device="cuda")
            reps = max(copies, 8)

            def run(op=op, xs=xs, rs=rs, q=q, sc=sc, reps=reps, copies=copies):
                for r in range(reps):
                    x = xs[r % copies]
                    if op == "rms_norm_dynamic_per_token_quant":
                        lq.rms_norm_dynamic_per_token_quant("fp8_dynamic", x, w, 1e-6, residual=rs[r % copies],
                                                            q=q, scales=sc, stream=stream)
                    elif op == "rms_norm_per_block_quant":
                        lq.rms_norm_per_block_quant(x, w, 1e-6, residual=rs[r % copies], q=q, scales=sc,
                                                    stream=stream)
                    elif op == "silu_and_mul_dynamic_per_token_quant":
                        lq.silu_and_mul_dynamic_per_token_quant("fp8_dynamic", x, q=q, scales=sc, stream=stream)
                    else:
                        lq.silu_and_mul_per_block_quant(x, q=q, scales=sc, stream=stream)
            g = capture(run, stream)
            time_replays(g, 3, stream)
            ms = time_replays(g, 10, stream) / (10 * reps)
            b = producer_bytes(op, M, cols, residual=rms)
            out.append({"op": op, "M": M, "K": cols, "residual": rms, "us": round(ms * 1e3, 3),
                        "GB/s": round(b / (ms * 1e-3) / 1e9, 1),
                        "frac_hbm": round(b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3), "bytes": b})
            del g, xs, rs
    return out


def moe_measurements(peaks, stream) -> list:
    """Per-call time of lq_grouped_scaled_mm on the Qwen3-30B-A3B expert
    GEMMs (128 experts, 8 per token) at decode batch sizes, graph-replayed
    over several seeded routings so that more than 2 x L2 of expert weights
    streams between two reads of one expert; beside it, the same work as one
    lq_scaled_mm per active expert."""
    out = []
    l2 = 126 * 2 ** 20
    E, top_k = inputs.QWEN3_30B_A3B_NUM_EXPERTS, inputs.QWEN3_30B_A3B_TOP_K
    g = torch.Generator().manual_seed(11)
    for layer, (K, N) in inputs.QWEN3_30B_A3B_EXPERTS.items():
        B = (torch.randint(0, 256, (E, N, K), generator=g, dtype=torch.uint8) & 0x77).cuda()   # finite e4m3 codes
        sb = (torch.rand((E, N), generator=g) * 1e-3).cuda()
        for tokens in (1, 8, 32, 64):
            T = tokens * top_k
            routes, nbytes = [], []
            while sum(nbytes) < 2 * l2 or len(routes) < 4:
                c = inputs.expert_counts(tokens, E, top_k, seed=inputs.stable_seed("moe-bench", layer, tokens, len(routes)))
                off = torch.tensor(np.concatenate([[0], np.cumsum(c)]), dtype=torch.int32).cuda()
                act = int((c > 0).sum())
                routes.append((off, act, c))
                nbytes.append(act * N * K + T * K + 4 * T + 4 * act * N + 2 * T * N)
            A = (torch.randint(0, 256, (T, K), generator=g, dtype=torch.uint8) & 0x77).cuda()
            sa = (torch.rand(T, generator=g) * 1e-2).cuda()
            C = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")

            def grouped(routes=routes, A=A, sa=sa, B=B, sb=sb, C=C):
                for off, _, _ in routes:
                    lq.grouped_scaled_mm("fp8_dynamic", A, sa, B, sb, off, C=C, stream=stream)

            def per_expert(routes=routes, A=A, sa=sa, B=B, sb=sb, C=C):
                for _, _, c in routes:
                    lo = 0
                    for e in range(E):
                        n = int(c[e])
                        if n:
                            lq.scaled_mm("fp8_dynamic", A[lo:lo + n], sa[lo:lo + n], B[e], sb[e], C[lo:lo + n],
                                         stream=stream)
                        lo += n

            row = {"layer": layer, "K": K, "N": N, "tokens": tokens, "T": T,
                   "active_experts": round(sum(a for _, a, _ in routes) / len(routes), 1)}
            for name, fn in (("grouped", grouped), ("per_expert_calls", per_expert)):
                gr = capture(fn, stream)
                time_replays(gr, 2, stream)
                ms = time_replays(gr, 5, stream) / (5 * len(routes))
                row[name + "_us"] = round(ms * 1e3, 2)
                del gr
            b = sum(nbytes) / len(nbytes)
            row["GB/s"] = round(b / (row["grouped_us"] * 1e-6) / 1e9, 1)
            row["frac_hbm"] = round(row["GB/s"] / peaks["hbm_gbs"], 3)
            out.append(row)
        del B
    return out


def capture(fn, stream) -> torch.cuda.CUDAGraph:
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()   # eager run once (allocations, lazy module loads)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


def time_cycle(graphs, n: int, stream) -> float:
    """Total ms of n graph launches cycling through `graphs`, CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(n):
            graphs[i % len(graphs)].replay()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def time_replays(g: torch.cuda.CUDAGraph, n: int, stream, pre=None, post=None) -> float:
    """Total ms of n replays, measured with CUDA events on `stream`."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(n):
            if pre:
                pre()
            g.replay()
            if post:
                post()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


# ----------------------------------------------------------- CPU leg
def _oracle_quant_weight(fmt: str, w):
    from oracle import lq_oracle as O
    from oracle import ue8m0_oracle as U
    if fmt == "block_fp8":
        return O.quant_weight_block128(w)
    if fmt == "block_fp8_ue8m0":
        return U.quant_weight_block128_ue8m0(w)
    return O.quant_per_channel(w, fmt)


def _oracle_step(fmt: str, x, qb, sb) -> None:
    """Quantize activations and compute the exact product, with the oracle."""
    from oracle import lq_oracle as O
    from oracle import ue8m0_oracle as U
    if fmt == "block_fp8":
        qa, sa = O.quant_per_token_group128(x)
        O.blockwise_ref(qa, sa, qb, sb)
    elif fmt == "block_fp8_ue8m0":
        qa, sa = U.quant_per_token_group128_ue8m0(x)
        U.blockwise_ue8m0_ref(qa, sa, qb, sb)
    else:
        qa, sa = O.quant_per_token(x, fmt)
        O.scaled_mm_ref(fmt, qa, sa, qb, sb)


def cpu_baseline(config: str, budget_s: float = 20.0) -> dict:
    """The oracle, as it stands, on a bounded sample of the same workload:
    every linear at the middle decode size (activation quantization plus the
    exact product), repeated until about `budget_s` seconds have passed, once
    on one core and once on every host core (output columns split over
    worker processes).  `value` and `cores` are the all-core figures."""
    from oracle import parallel_runner

    fmt, layers, ms = CONFIGS[config]
    M = ms[len(ms) // 2]
    prepared = []
    for layer, (K, N) in layers.items():
        w = inputs.weights(N, K, seed=inputs.stable_seed(config, "W", layer, 0)).float().numpy()
        qb, sb = _oracle_quant_weight(fmt, w)
        x = inputs.activations(M, K, seed=inputs.stable_seed(config, "A", layer, M, 0)).float().numpy()
        prepared.append((M, N, K, x, qb, sb))
    round_bytes = sum(gemm_bytes(fmt, M_, N, K) + quant_bytes(fmt, M_, K) for (M_, N, K, _, _, _) in prepared)
    t0 = time.perf_counter()
    rounds = 0
    while True:
        for (_, _, _, x, qb, sb) in prepared:
            _oracle_step(fmt, x, qb, sb)
        rounds += 1
        if time.perf_counter() - t0 > budget_s / 2 or rounds >= 50:
            break
    dt1 = time.perf_counter() - t0
    single = rounds * round_bytes / dt1 / 1e9
    box_cores = os.cpu_count() or 1
    par = parallel_runner.time_all_cores(fmt, [(x, qb, sb) for (_, _, _, x, qb, sb) in prepared], budget_s / 2)
    value = par["rounds"] * round_bytes / par["seconds"] / 1e9
    return {"value": value, "unit": "GB/s", "cores": par["workers"], "kind": "oracle",
            "single_core": {"value": single, "unit": "GB/s", "cores": 1, "rounds": rounds,
                            "seconds": round(dt1, 2)},
            "box_cores": box_cores,
            "sample": f"{config}: all {len(layers)} linears at M={M}, quantize + exact product; all-core: "
                      f"{par['rounds']} round(s) in {par['seconds']:.1f} s, output columns split into "
                      f"{par['tasks_per_round']} slices over {par['workers']} worker processes (numpy int64 "
                      f"matmul is single-threaded); single core: {rounds} round(s) in {dt1:.1f} s"}


def run_reference(args) -> None:
    """The oracle as the reference arm: each step quantizes one Qwen3 linear's
    activations at the middle decode size and computes the exact product for
    the first n output channels, n sized so that the whole --steps/--warmup
    run takes about two minutes of host time.  Throughput is the algorithmic
    bytes of the computed part over its time."""
    import numpy as np
    from oracle import lq_oracle as O

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = args.config
    fmt, layers, ms = CONFIGS[cfg]
    M = ms[len(ms) // 2]
    names = list(layers)
    total_steps = max(1, args.steps + args.warmup)
    budget = min(30.0, max(0.05, 120.0 / total_steps))       # seconds of oracle work per step
    prepared = {}
    for layer in names:
        K, N = layers[layer]
        n_max = min(N, 2048)   # weights are pre-quantized (not part of a step)
        w = inputs.weights(n_max, K, seed=inputs.stable_seed(cfg, "W", layer, 0)).float().numpy()
        x = inputs.activations(M, K, seed=inputs.stable_seed(cfg, "A", layer, M, 0)).float().numpy()
        qw = _oracle_quant_weight(fmt, w)
        prepared[layer] = (K, N, x, qw, n_max)

    def one(layer, n_cols):
        K, N, x, (qw, sw), _ = prepared[layer]
        qb = qw[:n_cols]
        sb = sw[:n_cols // 128] if fmt in BLOCK_FMTS else sw[:n_cols]
        t0 = time.perf_counter()
        _oracle_step(fmt, x, qb, sb)
        return time.perf_counter() - t0, gemm_bytes(fmt, M, n_cols, K) + quant_bytes(fmt, M, K)

    # calibrate columns per second on each layer, then size every step to the budget
    cols = {}
    for layer in names:
        n_max = prepared[layer][4]
        dt, _ = one(layer, 128)
        per_col = dt / 128
        cols[layer] = max(128, int(min(n_max, budget / max(per_col, 1e-9))) // 128 * 128)
    for i in range(args.warmup):
        one(names[i % len(names)], cols[names[i % len(names)]])
    nbytes, secs = 0, 0.0
    for i in range(args.steps):
        layer = names[i % len(names)]
        dt, b = one(layer, cols[layer])
        secs += dt
        nbytes += b
    value = nbytes / secs / 1e9
    lo, hi = min(cols.values()), max(cols.values())
    sample = (f"{cfg}: per step one linear (cycling {','.join(names)}) at M={M}, exact product for the first "
              f"{lo if lo == hi else f'{lo}-{hi}'} output channels; numpy int64 matmul, single thread")
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE[fmt],
           "data": "synthetic", "config": {"workload": cfg, "sample": sample},
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


METRIC = "scaled_mm HBM GB/s (algorithmic bytes) at M=1..32 on Qwen3 linear shapes"
DTYPE = {"fp8_dynamic": "e4m3 x e4m3 -> f32", "w8a8_int8": "s8 x s8 -> s32", "block_fp8": "e4m3 x e4m3 -> f32",
         "block_fp8_ue8m0": "e4m3 x e4m3 (UE8M0 block scales) -> f32"}


# ---------------------------------------------------------------- main
def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="lq", choices=["lq", "reference"])
    ap.add_argument("--copies", type=int, default=3, help="weight copies rotated to defeat L2 reuse")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-shape-reps", type=int, default=30)
    ap.add_argument("--no-producers", action="store_true",
                    help="skip the per-call timing of the producer-side fused quantizers")
    ap.add_argument("--no-moe", action="store_true", help="skip the grouped (MoE) GEMM timing")
    ap.add_argument("--ms", default=None,
                    help="comma-separated subset of the configuration's token counts (e.g. to profile one shape)")
    ap.add_argument("--layers", default=None, help="comma-separated subset of the configuration's linears")
    ap.add_argument("--path", default="separate", choices=["fused", "separate"],
                    help="fused: one lq_quant_scaled_mm per linear (quantization inside the GEMM kernel); "
                         "separate: lq_quant_per_token then lq_scaled_mm")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    lq.init_device(local)
    # the weights are quantized once, before any timed work, and never written afterwards
    lq.declare_static_weights(True)
    peaks = load_peaks()

    wl = Workload(args.config, device, copies=args.copies,
                  ms=[int(m) for m in args.ms.split(",")] if args.ms else None,
                  layers=args.layers.split(",") if args.layers else None)
    if not wl.calls:
        raise SystemExit("--ms / --layers leave no call of the configuration")
    stream = torch.cuda.Stream(device=device)
    stream.wait_stream(torch.cuda.current_stream())

    # one CUDA graph per step (quant + GEMM of every call), and GEMM-only / quant-only graphs
    use_fused = args.path == "fused" and wl.fmt not in BLOCK_FMTS
    if use_fused:
        lq.set_fuse_limit(1 << 40)   # every fusable call takes the one-kernel path
    g_step = capture(lambda: wl.step(stream, fused=use_fused), stream)
    g_gemm = capture(lambda: wl.step(stream, quant=False), stream)
    g_quant = capture(lambda: wl.step(stream, gemm=False), stream)

    sampler = ClockSampler(local)
    sampler.start()
    # warm-up, kept running for at least ~1 s so that clocks settle under load
    t_warm = time.perf_counter()
    time_replays(g_step, args.warmup, stream)
    while time.perf_counter() - t_warm < 1.0:
        time_replays(g_step, 20, stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms_total = time_replays(g_step, args.steps, stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = max_over_ranks(ms_total, device)
    ms_step = ms_total / args.steps

    step_bytes = wl.gemm_bytes + wl.quant_bytes
    value = aggregate_throughput(step_bytes, args.steps, ms_total, world) / 1e9
    tflops = aggregate_throughput(wl.flops, args.steps, ms_total, world) / 1e12

    # dominant kernel: scaled_mm, all launches of a step, timed on its own
    n_gemm_reps = max(50, min(args.steps, 500))
    time_replays(g_gemm, 10, stream)
    ms_gemm = time_replays(g_gemm, n_gemm_reps, stream) / n_gemm_reps
    time_replays(g_quant, 10, stream)
    ms_quant = time_replays(g_quant, n_gemm_reps, stream) / n_gemm_reps
    gemm_gbs = wl.gemm_bytes / (ms_gemm * 1e-3) / 1e9

    # per-shape breakdown: R calls of one shape per graph, rotating weight copies
    compute_bound = min(wl.ms) >= 256        # prefill configs: tensor-bound
    tensor_peak, tensor_peak_source = tensor_peak_8bit(wl.fmt, peaks)
    per_shape = []
    for c in wl.calls:
        reps = max(args.per_shape_reps, len(wl.weights[c["layer"]]))

        def one(c=c, reps=reps):
            for r in range(reps):
                wl.gemm(c, stream, copy=r)
        g = capture(one, stream)
        time_replays(g, 3, stream)
        ms = time_replays(g, 10, stream) / (10 * reps)
        del g
        # the same calls without programmatic dependent launch
        v_off = lq.make_variant(**{**c["variant"].as_dict(), "pdl": 0})

        def one_off(c=c, reps=reps, v_off=v_off):
            for r in range(reps):
                wl.gemm(c, stream, copy=r, variant=v_off)
        g = capture(one_off, stream)
        time_replays(g, 3, stream)
        ms_off = time_replays(g, 10, stream) / (10 * reps)
        del g
        # launch floor: every call its own graph launch (R = 1), weight copies still rotated
        n_copies = len(wl.weights[c["layer"]])
        singles = [capture(lambda c=c, r=r: wl.gemm(c, stream, copy=r), stream) for r in range(n_copies)]
        time_cycle(singles, 2 * n_copies, stream)
        n_single = max(30, 2 * n_copies)
        ms_single = time_cycle(singles, n_single, stream) / n_single
        del singles
        b = gemm_bytes(wl.fmt, c["M"], c["N"], c["K"])
        per_shape.append({"layer": c["layer"], "M": c["M"], "N": c["N"], "K": c["K"], "us": round(ms * 1e3, 3),
                          "GB/s": round(b / (ms * 1e-3) / 1e9, 1), "TFLOP/s": round(2 * c["M"] * c["N"] * c["K"] / (ms * 1e-3) / 1e12, 2),
                          "frac_hbm": round(b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                          "frac_tensor": round(2 * c["M"] * c["N"] * c["K"] / (ms * 1e-3) / 1e12 / tensor_peak, 3),
                          "us_pdl_off": round(ms_off * 1e3, 3), "us_single_graph": round(ms_single * 1e3, 3),
                          "variant": c["variant"].as_dict()})

    producers = producer_measurements(peaks, stream) if not args.no_producers else []
    moe = moe_measurements(peaks, stream) if not args.no_moe else []

    # End to end through the public API: every step copies its activations
    # host->device from pinned memory, runs, and copies every output back.
    # Two buffer sets and two copy streams let the copies of neighbouring
    # steps overlap the current step's kernels (PCIe is full duplex).
    x_bufs = [wl.x_all, torch.empty_like(wl.x_all)]
    c_bufs = [wl.c_all, torch.empty_like(wl.c_all)]
    c_host = [wl.c_host, torch.empty(wl.c_all.shape, dtype=torch.bfloat16, pin_memory=True)]
    g_e2e = []
    for b in range(2):
        wl.bind(x_bufs[b], c_bufs[b])
        g_e2e.append(capture(lambda: wl.step(stream, fused=use_fused), stream))
    wl.bind(x_bufs[0], c_bufs[0])
    h2d_s = torch.cuda.Stream(device=device)
    d2h_s = torch.cuda.Stream(device=device)

    def run_e2e(n: int) -> float:
        ev_h2d = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_d2h = [torch.cuda.Event() for _ in range(2)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(h2d_s)
        stream.wait_stream(h2d_s)
        d2h_s.wait_stream(h2d_s)
        for i in range(n):
            b = i % 2
            if i >= 2:
                h2d_s.wait_event(ev_comp[b])          # step i-2 no longer reads x_bufs[b]
            with torch.cuda.stream(h2d_s):
                x_bufs[b].copy_(wl.x_host, non_blocking=True)
            ev_h2d[b].record(h2d_s)
            stream.wait_event(ev_h2d[b])
            if i >= 2:
                stream.wait_event(ev_d2h[b])          # c_bufs[b] of step i-2 has been copied out
            with torch.cuda.stream(stream):
                g_e2e[b].replay()
            ev_comp[b].record(stream)
            d2h_s.wait_event(ev_comp[b])
            with torch.cuda.stream(d2h_s):
                c_host[b].copy_(c_bufs[b], non_blocking=True)
            ev_d2h[b].record(d2h_s)
        stream.wait_stream(d2h_s)
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end)

    run_e2e(4)
    e2e_n = max(20, min(args.steps, 500))
    ms_e2e = run_e2e(e2e_n) / e2e_n
    e2e_val = world * step_bytes / (ms_e2e * 1e-3) / 1e9
    del g_e2e

    del g_step, g_gemm, g_quant
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(args.config, budget_s=15.0)

    layers = ",".join(f"{k}({K}x{N})" for k, (K, N) in wl.layers.items())
    if use_fused:
        # the dominant (and only) kernel of the step: the fused quantize + GEMM kernel
        roofline = {"bound": "hbm", "kernel": "lq_quant_scaled_mm fused kernel (all launches of one step)",
                    "achieved": round(value / world, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(value / world / peaks["hbm_gbs"], 4),
                    "traffic": recorded_traffic(args.config, "fused"),
                    "traffic_unit": "DRAM bytes per step of the fused launches (ncu)",
                    "algorithmic_bytes_per_step": step_bytes, "launches_per_step": wl.launches_per_step(fused=True),
                    "us_per_step": round(ms_step * 1e3, 2), "peak_source": peaks["source"]}
    elif compute_bound:
        # prefill: 2MNK flops against the 8-bit tensor-core peak (a kernel timed inside a long step:
        # the sustained bf16 measurement times the nominal 8-bit / bf16 ratio of 2)
        gemm_tflops = wl.flops / (ms_gemm * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": "scaled_mm (all launches of one step)",
                    "achieved": round(gemm_tflops, 1), "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
                    "frac": round(gemm_tflops / tensor_peak, 4),
                    "traffic": recorded_traffic(args.config, "scaled_mm"),
                    "traffic_unit": "DRAM bytes per step of scaled_mm launches (ncu)",
                    "algorithmic_flops_per_step": wl.flops, "launches_per_step": wl.launches_per_step(quant=False),
                    "us_per_step": round(ms_gemm * 1e3, 2),
                    "peak_source": tensor_peak_source}
    else:
        roofline = {"bound": "hbm", "kernel": "scaled_mm (all launches of one step)",
                    "achieved": round(gemm_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(gemm_gbs / peaks["hbm_gbs"], 4),
                    "traffic": recorded_traffic(args.config, "scaled_mm"),
                    "traffic_unit": "DRAM bytes per step of scaled_mm launches (ncu)",
                    "algorithmic_bytes_per_step": wl.gemm_bytes, "launches_per_step": wl.launches_per_step(quant=False),
                    "us_per_step": round(ms_gemm * 1e3, 2), "peak_source": peaks["source"]}
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE[wl.fmt],
        "data": "synthetic",
        "config": {"workload": args.config + ("" if not (args.ms or args.layers) else " (subset)"),
                   "format": wl.fmt, "layers": layers, "M": list(wl.ms),
                   "calls_per_step": len(wl.calls), "parallelism": f"replicas x{world}",
                   "l2": "weight copies rotated so that > 2x L2 is streamed between two reads of one copy",
                   "graph": "one CUDA graph per step",
                   "path": "lq_quant_scaled_mm (activation quantization fused into the GEMM kernel)" if use_fused
                   else "lq_quant_per_token + lq_scaled_mm"},
        "tflops": round(tflops, 3),
        "frac_hbm_step": round(value / world / peaks["hbm_gbs"], 4),
        "roofline": roofline,
        "scaled_mm_only": {"GB/s": round(gemm_gbs, 1), "frac": round(gemm_gbs / peaks["hbm_gbs"], 4),
                           "us_per_step": round(ms_gemm * 1e3, 2), "algorithmic_bytes_per_step": wl.gemm_bytes,
                           "what": f"the step's {len(wl.calls)} lq_scaled_mm calls alone (codes already quantized)"},
        "quant_us_per_step": round(ms_quant * 1e3, 2),
        "clocks": clocks,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "ms_per_step": round(ms_e2e, 5),
                "pipeline": "H2D / step / D2H on three streams, double-buffered",
                "h2d_bytes_per_step": wl.x_all.numel() * 2, "d2h_bytes_per_step": wl.c_all.numel() * 2},
        "gpu_launches": wl.launches_per_step(fused=use_fused) * args.steps,
        "per_shape": per_shape,
        "producers": producers,
        "moe": moe,
    }
    if cpu is not None:
        out["cpu_baseline"] = cpu
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
