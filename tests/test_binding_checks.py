"""The Python binding's argument checks, on the CPU: every tensor argument
is checked (dtype, rank, contiguity, exact shape, one device) before the C
function is called, so that a wrongly sized scale or output tensor is refused
instead of being read or written out of bounds by a kernel.  The library is
replaced by a recorder and the device type by the CPU; nothing here launches
anything."""

import types

import pytest
import torch

from quantized_linear_gemm_b200 import lq

S = types.SimpleNamespace(cuda_stream=0)   # a stream handle for the recorder


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(lq, "_DEVICE_TYPE", "cpu")
    monkeypatch.setattr(lq, "lib", lambda: r)
    return r


def _codes(*shape, dtype=torch.uint8):
    return torch.zeros(shape, dtype=dtype)


def _f32(*shape):
    return torch.ones(shape, dtype=torch.float32)


def test_scaled_mm_accepts_the_documented_layouts(rec):
    M, N, K = 5, 256, 384
    C = lq.scaled_mm("fp8_dynamic", _codes(M, K), _f32(M), _codes(N, K), _f32(N), stream=S)
    assert C.shape == (M, N) and C.dtype == torch.bfloat16
    name, args = rec.calls[-1]
    assert name == "lq_scaled_mm" and args[0] == lq.FP8_DYNAMIC and args[6:9] == (M, N, K)
    lq.scaled_mm("block_fp8", _codes(M, K), _f32(M, K // 128), _codes(N, K), _f32(N // 128, K // 128), stream=S)
    lq.scaled_mm("block_fp8_ue8m0", _codes(M, K), _codes(M, K // 128), _codes(N, K),
                 _codes(N // 128, K // 128), stream=S)
    lq.scaled_mm("w8a8_int8", _codes(M, K, dtype=torch.int8), _f32(M), _codes(N, K, dtype=torch.int8), _f32(N),
                 stream=S)
    assert len(rec.calls) == 4


def test_degenerate_sizes_are_accepted(rec):
    lq.scaled_mm("fp8_dynamic", _codes(0, 128), _f32(0), _codes(16, 128), _f32(16), stream=S)   # M = 0
    lq.scaled_mm("fp8_dynamic", _codes(4, 0), _f32(4), _codes(16, 0), _f32(16), stream=S)       # K = 0
    lq.quant_per_token("fp8_dynamic", torch.zeros((0, 64), dtype=torch.bfloat16), stream=S)
    assert len(rec.calls) == 3


@pytest.mark.parametrize("case", ["a_short", "b_long", "block_a_wide", "block_b_transposed", "C_shape", "K"])
def test_scaled_mm_refuses_wrong_shapes(rec, case):
    M, N, K = 5, 256, 384
    fmt, A, sa, B, sb, C = "fp8_dynamic", _codes(M, K), _f32(M), _codes(N, K), _f32(N), None
    if case == "a_short":
        sa = _f32(M - 1)
    elif case == "b_long":
        sb = _f32(N + 8)
    elif case == "block_a_wide":
        fmt, sa, sb = "block_fp8", _f32(M, K // 128 + 1), _f32(N // 128, K // 128)
    elif case == "block_b_transposed":
        fmt, sa, sb = "block_fp8", _f32(M, K // 128), _f32(K // 128, N // 128)
    elif case == "C_shape":
        C = torch.empty((M, N + 8), dtype=torch.bfloat16)
    elif case == "K":
        B = _codes(N, K + 16)
    with pytest.raises(ValueError):
        lq.scaled_mm(fmt, A, sa, B, sb, C=C, stream=S)
    assert rec.calls == []


def test_scaled_mm_refuses_wrong_dtypes(rec):
    M, N, K = 5, 256, 384
    with pytest.raises(TypeError):   # UE8M0 scales are bytes
        lq.scaled_mm("block_fp8_ue8m0", _codes(M, K), _f32(M, K // 128), _codes(N, K), _f32(N // 128, K // 128),
                     stream=S)
    with pytest.raises(TypeError):   # fp32 scales, not fp16
        lq.scaled_mm("fp8_dynamic", _codes(M, K), torch.ones(M, dtype=torch.float16), _codes(N, K), _f32(N),
                     stream=S)
    with pytest.raises(ValueError):  # non-contiguous codes
        lq.scaled_mm("fp8_dynamic", _codes(K, M).t(), _f32(M), _codes(N, K), _f32(N), stream=S)
    assert rec.calls == []


def test_bias_and_fused_and_i32acc_checks(rec):
    M, N, K = 3, 128, 256
    A, B = _codes(M, K), _codes(N, K)
    lq.scaled_mm_bias("fp8_dynamic", A, _f32(M), B, _f32(N), torch.zeros(N, dtype=torch.bfloat16), stream=S)
    with pytest.raises(ValueError):
        lq.scaled_mm_bias("fp8_dynamic", A, _f32(M), B, _f32(N), torch.zeros(N - 8, dtype=torch.bfloat16), stream=S)
    with pytest.raises(ValueError):   # the scales are checked here too
        lq.scaled_mm_bias("fp8_dynamic", A, _f32(M + 1), B, _f32(N), torch.zeros(N, dtype=torch.bfloat16), stream=S)
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    lq.quant_scaled_mm("fp8_dynamic", x, B, _f32(N), stream=S)
    with pytest.raises(ValueError):
        lq.quant_scaled_mm("fp8_dynamic", x, B, _f32(N), s=_f32(M + 1), stream=S)
    with pytest.raises(ValueError):
        lq.quant_scaled_mm("fp8_dynamic", x, B, _f32(N), q=_codes(M, K - 16), stream=S)
    Ai, Bi = _codes(M, K, dtype=torch.int8), _codes(N, K, dtype=torch.int8)
    lq.scaled_mm_i32acc(Ai, _f32(M), Bi, _f32(N), stream=S)
    with pytest.raises(ValueError):
        lq.scaled_mm_i32acc(Ai, _f32(M), Bi, _f32(N), acc=torch.empty((M, N - 8), dtype=torch.int32), stream=S)
    assert [c[0] for c in rec.calls] == ["lq_scaled_mm_bias", "lq_quant_scaled_mm", "lq_scaled_mm_i32acc"]


def test_grouped_checks(rec):
    T, E, N, K = 20, 3, 256, 512
    A, B = _codes(T, K), _codes(E, N, K)
    off = torch.tensor([0, 10, 15, 20], dtype=torch.int32)
    C = lq.grouped_scaled_mm("fp8_dynamic", A, _f32(T), B, _f32(E, N), off, stream=S)
    assert C.shape == (T, N)
    for bad in (dict(off=off[:3]), dict(sb=_f32(E * N)), dict(sa=_f32(T - 1)), dict(B=_codes(E, N, K + 16))):
        with pytest.raises(ValueError):
            lq.grouped_scaled_mm("fp8_dynamic", A, bad.get("sa", _f32(T)), bad.get("B", B), bad.get("sb", _f32(E, N)),
                                 bad.get("off", off), stream=S)
    assert len(rec.calls) == 1


def test_quantizer_output_checks(rec):
    M, K = 4, 256
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    q, s = lq.quant_per_token("w8a8_int8", x, stream=S)
    assert q.dtype == torch.int8 and s.shape == (M,)
    q, s = lq.quant_per_token_group128(x, stream=S)
    assert s.shape == (M, K // 128)
    with pytest.raises(ValueError):
        lq.quant_per_token("fp8_dynamic", x, q=_codes(M, K), scales=_f32(M, 1), stream=S)
    with pytest.raises(TypeError):
        lq.quant_per_token_group128_ue8m0(x, scales=_f32(M, K // 128), stream=S)
    with pytest.raises(ValueError):
        lq.quant_weight_block128(torch.zeros((256, K), dtype=torch.bfloat16), scales=_f32(1, 2), stream=S)
    w = torch.ones(K, dtype=torch.bfloat16)
    lq.rms_norm_dynamic_per_token_quant("fp8_dynamic", x, w, 1e-6, stream=S)
    with pytest.raises(ValueError):
        lq.rms_norm_per_block_quant(x, torch.ones(K - 128, dtype=torch.bfloat16), 1e-6, stream=S)
    with pytest.raises(ValueError):
        lq.rms_norm_dynamic_per_token_quant("fp8_dynamic", x, w, 1e-6, residual=torch.zeros((M, K - 16),
                                                                                             dtype=torch.bfloat16),
                                            stream=S)
    with pytest.raises(ValueError):
        lq.silu_and_mul_per_block_quant(torch.zeros((M, 255), dtype=torch.bfloat16), stream=S)
    assert [c[0] for c in rec.calls] == ["lq_quant_per_token", "lq_quant_per_token_group128",
                                         "lq_rms_norm_dynamic_per_token_quant"]


def test_trace_buffer_checks(rec):
    lq.set_trace(torch.zeros(12 * 4, dtype=torch.int64))
    lq.set_trace(None)
    with pytest.raises(TypeError):
        lq.set_trace(torch.zeros(48, dtype=torch.int32))
    with pytest.raises(ValueError):
        lq.set_trace(torch.zeros((4, 12), dtype=torch.int64))
    assert [c[0] for c in rec.calls] == ["lq_set_trace", "lq_set_trace"]


def test_tensors_must_share_one_device():
    a = torch.zeros(4)
    with pytest.raises(ValueError):
        lq._one_device(a, torch.zeros(4, device="meta"))
    lq._one_device(a, None, torch.zeros(2))


def test_cpu_tensors_are_refused_by_default():
    """Without the recorder the binding takes GPU tensors only: a host pointer
    never reaches a kernel."""
    with pytest.raises(ValueError):
        lq.scaled_mm("fp8_dynamic", _codes(1, 16), _f32(1), _codes(8, 16), _f32(8), stream=S)
