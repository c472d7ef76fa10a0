"""The JSON line of bench.py, on the CPU: every key the benchmark contract
asks for is present and well formed.  bench.py runs in a subprocess in which
the library is a recorder that launches nothing (every call returns LQ_OK)
and torch's CUDA calls are CPU stand-ins, so the numbers are meaningless;
what is checked is the shape of the line (and that the binding accepts every
call the benchmark makes).  The reference arm runs for real: it is the CPU
oracle."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# CPU stand-ins for the CUDA calls bench.py makes, then bench.py itself.
_RUNNER = r'''
import contextlib, functools, sys, types
import torch

def _cpu(d):
    if isinstance(d, str) and d.startswith("cuda"): return "cpu"
    if isinstance(d, torch.device) and d.type == "cuda": return torch.device("cpu")
    return d

def _wrap(fn):
    @functools.wraps(fn)
    def w(*a, **k):
        if "device" in k: k["device"] = _cpu(k["device"])
        k.pop("pin_memory", None)
        return fn(*a, **k)
    return w

for name in ("empty", "zeros", "ones", "full", "rand", "randn", "randint", "tensor", "arange", "empty_like",
             "zeros_like", "full_like", "as_tensor"):
    setattr(torch, name, _wrap(getattr(torch, name)))
_to = torch.Tensor.to
torch.Tensor.to = lambda self, *a, **k: _to(self, *[_cpu(x) for x in a], **{kk: _cpu(v) for kk, v in k.items()})
torch.Tensor.cuda = lambda self, *a, **k: self
torch.Tensor.pin_memory = lambda self, *a, **k: self

class _Any:
    cuda_stream = 0
    device = types.SimpleNamespace(index=0, type="cuda")
    def __init__(self, *a, **k): pass
    def elapsed_time(self, other): return 1.0
    def __getattr__(self, name): return lambda *a, **k: None

torch.cuda.is_available = lambda: True
torch.cuda.device_count = lambda: 1
torch.cuda.current_device = lambda: 0
torch.cuda.set_device = lambda *a, **k: None
torch.cuda.get_device_name = lambda *a: "stand-in"
torch.cuda.synchronize = lambda *a, **k: None
torch.cuda.empty_cache = lambda: None
torch.cuda.Stream = torch.cuda.Event = torch.cuda.CUDAGraph = _Any
torch.cuda.current_stream = lambda *a, **k: _Any()
torch.cuda.stream = lambda s: contextlib.nullcontext()
torch.cuda.graph = lambda *a, **k: contextlib.nullcontext()

from quantized_linear_gemm_b200 import lq

class _Recorder:
    def __getattr__(self, name):
        return (lambda *a: b"stand-in") if name == "lq_version" else (lambda *a: 0)

lq._DEVICE_TYPE = "cpu"
lq.lib = lambda: _Recorder()
import bench
_cpu_baseline = bench.cpu_baseline
bench.cpu_baseline = lambda config, budget_s=20.0: _cpu_baseline(config, budget_s=1.0)   # a short sample
sys.argv = ["bench.py"] + sys.argv[1:]
bench.main()
'''


def _run(args, stand_in=True, timeout=600):
    cmd = [sys.executable, "-c", _RUNNER] + args if stand_in else [sys.executable, "bench.py"] + args
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _common(d, cpu=True):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "e2e") + (("cpu_baseline",) if cpu else ()):
        assert k in d, k
    assert isinstance(d["config"], dict) and "workload" in d["config"]
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["data"] == "synthetic"
    assert d["warmup"] >= 3
    e = d["e2e"]
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(e)


@pytest.mark.slow
def test_bench_line_has_every_contract_key():
    d = _run(["--steps", "2", "--warmup", "3"])
    _common(d)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["config"]["workload"] == "qwen3-8b-fp8-decode"
    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3 * max(1.0, r["frac"])
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    assert isinstance(d["gpu_launches"], int) and d["gpu_launches"] > 0
    assert len(d["per_shape"]) == 28
    for p in d["per_shape"]:
        assert {"us", "GB/s", "frac_hbm", "us_pdl_off", "us_single_graph", "variant"} <= set(p)
    assert d["producers"] and d["moe"]


@pytest.mark.slow
def test_prefill_line_reports_a_tensor_roofline():
    d = _run(["--config", "qwen3-32b-fp8-prefill", "--steps", "1", "--warmup", "3", "--no-cpu-baseline",
              "--no-producers", "--no-moe", "--per-shape-reps", "1"])
    _common(d, cpu=False)
    assert d["roofline"]["bound"] == "tensor" and d["roofline"]["unit"] == "TFLOP/s"
    assert all("frac_tensor" in p for p in d["per_shape"])


@pytest.mark.slow
def test_reference_arm_line():
    """The reference arm is the CPU oracle itself (no stand-ins)."""
    d = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"], stand_in=False)
    _common(d)
    assert d["impl"] == "reference"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
