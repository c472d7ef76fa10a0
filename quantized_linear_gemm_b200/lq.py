"""Python binding of liblq (ctypes).  Argument marshalling only.

Every function here checks its tensors (dtype, rank, contiguity, the exact
shape the C function reads or writes, and one device: the current CUDA
device), then calls the C function of the same name in ``liblq.so`` on
torch's current CUDA stream.  All arithmetic runs in the library's CUDA kernels; there is no
fallback.  If ``liblq.so`` is missing the first call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblq.so")

FP8_DYNAMIC = 0
W8A8_INT8 = 1
BLOCK_FP8 = 2
BLOCK_FP8_UE8M0 = 3
FORMATS = {"fp8_dynamic": FP8_DYNAMIC, "w8a8_int8": W8A8_INT8, "block_fp8": BLOCK_FP8,
           "block_fp8_ue8m0": BLOCK_FP8_UE8M0}

STATUS = {
    0: "LQ_OK", 1: "LQ_ERR_INVALID_ARG", 2: "LQ_ERR_ALIGNMENT", 3: "LQ_ERR_UNSUPPORTED_SHAPE",
    4: "LQ_ERR_WORKSPACE", 5: "LQ_ERR_CUDA", 6: "LQ_ERR_DEVICE_TIMEOUT", 7: "LQ_ERR_TABLE",
}

# every symbol that include/lq.h declares
EXPORTED = (
    "lq_scaled_mm", "lq_scaled_mm_i32acc", "lq_quant_per_token", "lq_quant_per_token_group128",
    "lq_quant_weight_block128", "lq_select_variant", "lq_load_dispatch_table", "lq_dispatch_table_size",
    "lq_init_device", "lq_reserve_workspace", "lq_workspace_bytes", "lq_device_status",
    "lq_status_string", "lq_version", "lq_set_trace", "lq_scaled_mm_noalloc", "lq_test_inject_stall",
    "lq_test_silu_bf16",
    "lq_quant_scaled_mm", "lq_set_fuse_limit", "lq_rms_norm_dynamic_per_token_quant",
    "lq_rms_norm_per_block_quant", "lq_silu_and_mul_dynamic_per_token_quant", "lq_silu_and_mul_per_block_quant",
    "lq_grouped_scaled_mm", "lq_quant_per_token_group128_ue8m0", "lq_quant_weight_block128_ue8m0",
    "lq_scaled_mm_bias", "lq_declare_static_weights",
)


class LQError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Variant(ctypes.Structure):
    _fields_ = [("swap_ab", ctypes.c_int32), ("split_k", ctypes.c_int32), ("tile_n", ctypes.c_int32),
                ("stages", ctypes.c_int32), ("reduce", ctypes.c_int32), ("pdl", ctypes.c_int32),
                ("persistent", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {f: int(getattr(self, f)) for f, _ in self._fields_}


def make_variant(swap_ab=0, split_k=1, tile_n=None, stages=0, reduce=1, pdl=1, persistent=0) -> Variant:
    if tile_n is None:
        tile_n = 32 if swap_ab else 128
    return Variant(int(swap_ab), int(split_k), int(tile_n), int(stages), int(reduce), int(pdl), int(persistent))


_lib = None
_lock = threading.Lock()

_vp, _i64, _i32, _st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """The loaded liblq.so (loaded on first use)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m quantized_linear_gemm_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            L.lq_scaled_mm.argtypes = [_i32, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.POINTER(Variant), _st]
            L.lq_quant_scaled_mm.argtypes = [_i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                             ctypes.POINTER(Variant), _st]
            L.lq_quant_scaled_mm.restype = _i32
            L.lq_scaled_mm_noalloc.argtypes = [_i32, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                               ctypes.POINTER(Variant), _st]
            L.lq_scaled_mm_noalloc.restype = _i32
            L.lq_scaled_mm_i32acc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                              ctypes.POINTER(Variant), _st]
            L.lq_quant_per_token.argtypes = [_i32, _vp, _vp, _vp, _i64, _i64, _st]
            L.lq_quant_per_token_group128.argtypes = [_vp, _vp, _vp, _i64, _i64, _st]
            L.lq_quant_weight_block128.argtypes = [_vp, _vp, _vp, _i64, _i64, _st]
            L.lq_select_variant.argtypes = [_i32, _i64, _i64, _i64, ctypes.POINTER(Variant)]
            L.lq_load_dispatch_table.argtypes = [ctypes.c_char_p]
            L.lq_dispatch_table_size.argtypes = []
            L.lq_dispatch_table_size.restype = _i64
            L.lq_init_device.argtypes = [_i32]
            L.lq_reserve_workspace.argtypes = [_i32, ctypes.c_size_t]
            L.lq_workspace_bytes.argtypes = [_i32, _i64, _i64, _i64, ctypes.POINTER(Variant)]
            L.lq_workspace_bytes.restype = ctypes.c_size_t
            L.lq_device_status.argtypes = [_i32]
            L.lq_status_string.argtypes = [_i32]
            L.lq_status_string.restype = ctypes.c_char_p
            L.lq_test_inject_stall.argtypes = [_i32, ctypes.c_uint64]
            L.lq_test_inject_stall.restype = _i32
            L.lq_test_silu_bf16.argtypes = [_vp, _vp, _i64, _vp]
            L.lq_test_silu_bf16.restype = _i32
            L.lq_set_trace.argtypes = [_vp]
            L.lq_set_trace.restype = _i32
            L.lq_declare_static_weights.argtypes = [_i32]
            L.lq_declare_static_weights.restype = _i32
            L.lq_set_fuse_limit.argtypes = [ctypes.c_int64]
            L.lq_set_fuse_limit.restype = ctypes.c_int64
            L.lq_rms_norm_dynamic_per_token_quant.argtypes = [_i32, _vp, _vp, _vp, ctypes.c_float, _vp, _vp,
                                                              _i64, _i64, _st]
            L.lq_rms_norm_per_block_quant.argtypes = [_vp, _vp, _vp, ctypes.c_float, _vp, _vp, _i64, _i64, _st]
            L.lq_silu_and_mul_dynamic_per_token_quant.argtypes = [_i32, _vp, _vp, _vp, _i64, _i64, _st]
            L.lq_silu_and_mul_per_block_quant.argtypes = [_vp, _vp, _vp, _i64, _i64, _st]
            for name in ("lq_rms_norm_dynamic_per_token_quant", "lq_rms_norm_per_block_quant",
                         "lq_silu_and_mul_dynamic_per_token_quant", "lq_silu_and_mul_per_block_quant"):
                getattr(L, name).restype = _i32
            L.lq_grouped_scaled_mm.argtypes = [_i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                               ctypes.POINTER(Variant), _st]
            L.lq_grouped_scaled_mm.restype = _i32
            for name in ("lq_quant_per_token_group128_ue8m0", "lq_quant_weight_block128_ue8m0"):
                getattr(L, name).argtypes = [_vp, _vp, _vp, _i64, _i64, _st]
                getattr(L, name).restype = _i32
            L.lq_scaled_mm_bias.argtypes = [_i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                            ctypes.POINTER(Variant), _st]
            L.lq_scaled_mm_bias.restype = _i32
            L.lq_version.argtypes = []
            L.lq_version.restype = ctypes.c_char_p
            for name in ("lq_scaled_mm", "lq_scaled_mm_i32acc", "lq_quant_per_token", "lq_quant_per_token_group128",
                         "lq_quant_weight_block128", "lq_select_variant", "lq_load_dispatch_table",
                         "lq_init_device", "lq_reserve_workspace", "lq_device_status"):
                getattr(L, name).restype = _i32
            _lib = L
    return _lib


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise LQError(fn, rc)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _fmt(fmt) -> int:
    if isinstance(fmt, str):
        return FORMATS[fmt]
    return int(fmt)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


_DEVICE_TYPE = "cuda"   # the only device type the library runs on

_CODE_DTYPES = (torch.uint8, torch.int8, torch.float8_e4m3fn)   # one byte per code


def _need(t: torch.Tensor, name: str, dtypes, ndim: int, shape=None) -> None:
    """t is a contiguous ndim-d tensor of one of `dtypes` on the GPU, of
    exactly `shape` when given (the C ABI reads that many elements)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.device.type != _DEVICE_TYPE:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _one_device(*ts) -> None:
    """All tensors on one device, the current CUDA device (the library
    launches on the current device and dereferences every pointer there)."""
    ts = [t for t in ts if t is not None]
    dev = ts[0].device
    for t in ts[1:]:
        if t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    if dev.type == "cuda" and dev.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {dev} but the current CUDA device is cuda:{torch.cuda.current_device()}")


def _scales_spec(f: int, M: int, N: int, K: int):
    """dtype and shapes of (a_scales, b_scales) for format f: per token and
    per output channel, or per 1 x 128 group and per 128 x 128 block."""
    if f in (BLOCK_FP8, BLOCK_FP8_UE8M0):
        dt = (torch.uint8,) if f == BLOCK_FP8_UE8M0 else (torch.float32,)
        return dt, (M, K // 128), (N // 128, K // 128)
    return (torch.float32,), (M,), (N,)


def _gemm_operands(f: int, A, a_scales, B, b_scales, C):
    """Check the operands of one [M, K] x [N, K]^T product; returns (M, N, K)."""
    _need(A, "A", _CODE_DTYPES, 2)
    _need(B, "B", _CODE_DTYPES, 2)
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("A and B disagree on K")
    dt, sa, sb = _scales_spec(f, M, N, K)
    _need(a_scales, "a_scales", dt, len(sa), sa)
    _need(b_scales, "b_scales", dt, len(sb), sb)
    if C is not None:
        _need(C, "C", (torch.bfloat16,), 2, (M, N))
    _one_device(A, a_scales, B, b_scales, C)
    return M, N, K


def _outputs(device, q, q_shape, q_dtype, scales, s_shape, s_dtype=torch.float32):
    """Allocate the codes / scales outputs, or check the caller's."""
    if q is None:
        q = torch.empty(q_shape, dtype=q_dtype, device=device)
    else:
        _need(q, "q", _CODE_DTYPES, len(q_shape), q_shape)
    if scales is None:
        scales = torch.empty(s_shape, dtype=s_dtype, device=device)
    else:
        _need(scales, "scales", (s_dtype,), len(s_shape), s_shape)
    return q, scales


def _code_dtype(f: int):
    return torch.int8 if f == W8A8_INT8 else torch.uint8


def scaled_mm(fmt, A: torch.Tensor, a_scales: torch.Tensor, B: torch.Tensor, b_scales: torch.Tensor,
              C: torch.Tensor | None = None, variant: Variant | None = None, stream=None) -> torch.Tensor:
    """C[M, N] (bf16) = dequant(A[M, K]) @ dequant(B[N, K])^T through ``lq_scaled_mm``."""
    f = _fmt(fmt)
    M, N, K = _gemm_operands(f, A, a_scales, B, b_scales, C)
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    rc = lib().lq_scaled_mm(f, _ptr(A), _ptr(a_scales), _ptr(B), _ptr(b_scales), _ptr(C), M, N, K,
                            ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_scaled_mm", rc)
    return C


def quant_scaled_mm(fmt, x: torch.Tensor, B: torch.Tensor, b_scales: torch.Tensor, C=None, q=None, s=None,
                    variant: Variant | None = None, stream=None):
    """``lq_quant_scaled_mm``: per-token quantization of bf16 ``x`` fused with
    scaled_mm.  Returns (C, codes, scales)."""
    f = _fmt(fmt)
    _need(x, "x", (torch.bfloat16,), 2)
    _need(B, "B", _CODE_DTYPES, 2)
    M, K = x.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("x and B disagree on K")
    _need(b_scales, "b_scales", (torch.float32,), 1, (N,))
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(C, "C", (torch.bfloat16,), 2, (M, N))
    q, s = _outputs(x.device, q, (M, K), _code_dtype(f), s, (M,))
    _one_device(x, B, b_scales, C, q, s)
    rc = lib().lq_quant_scaled_mm(f, _ptr(x), _ptr(B), _ptr(b_scales), _ptr(C), _ptr(q), _ptr(s), M, N, K,
                                  ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_quant_scaled_mm", rc)
    return C, q, s


def scaled_mm_bias(fmt, A: torch.Tensor, a_scales: torch.Tensor, B: torch.Tensor, b_scales: torch.Tensor,
                   bias: torch.Tensor, C: torch.Tensor | None = None, variant: Variant | None = None,
                   stream=None) -> torch.Tensor:
    """``lq_scaled_mm_bias``: scaled_mm plus a bf16 bias [N] added before the rounding."""
    f = _fmt(fmt)
    M, N, K = _gemm_operands(f, A, a_scales, B, b_scales, C)
    _need(bias, "bias", (torch.bfloat16,), 1, (N,))
    _one_device(A, bias)
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    rc = lib().lq_scaled_mm_bias(f, _ptr(A), _ptr(a_scales), _ptr(B), _ptr(b_scales), _ptr(bias), _ptr(C), M, N, K,
                                 ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_scaled_mm_bias", rc)
    return C


def grouped_scaled_mm(fmt, A: torch.Tensor, a_scales: torch.Tensor, B: torch.Tensor, b_scales: torch.Tensor,
                      expert_offsets: torch.Tensor, C: torch.Tensor | None = None, variant: Variant | None = None,
                      stream=None) -> torch.Tensor:
    """``lq_grouped_scaled_mm``: A [T, K] tokens sorted by expert, B [E, N, K]
    stacked expert weights, b_scales [E, N], expert_offsets int32 [E + 1] on
    the device.  Returns C [T, N] bf16."""
    f = _fmt(fmt)
    _need(A, "A", _CODE_DTYPES, 2)
    _need(B, "B", _CODE_DTYPES, 3)
    T, K = A.shape
    E, N, KB = B.shape
    if KB != K:
        raise ValueError("A and B disagree on K")
    _need(a_scales, "a_scales", (torch.float32,), 1, (T,))
    _need(b_scales, "b_scales", (torch.float32,), 2, (E, N))
    _need(expert_offsets, "expert_offsets", (torch.int32,), 1, (E + 1,))
    if C is None:
        C = torch.empty((T, N), dtype=torch.bfloat16, device=A.device)
    _need(C, "C", (torch.bfloat16,), 2, (T, N))
    _one_device(A, a_scales, B, b_scales, expert_offsets, C)
    rc = lib().lq_grouped_scaled_mm(f, _ptr(A), _ptr(a_scales), _ptr(B), _ptr(b_scales), _ptr(C),
                                    _ptr(expert_offsets), E, T, N, K,
                                    ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_grouped_scaled_mm", rc)
    return C


def scaled_mm_noalloc(fmt, A: torch.Tensor, a_scales: torch.Tensor, B: torch.Tensor, b_scales: torch.Tensor,
                      C: torch.Tensor | None = None, variant: Variant | None = None, stream=None) -> torch.Tensor:
    """``lq_scaled_mm_noalloc``: scaled_mm whose Split-K partials use the library's
    fixed device array instead of allocated workspace (see include/lq.h)."""
    f = _fmt(fmt)
    M, N, K = _gemm_operands(f, A, a_scales, B, b_scales, C)
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    rc = lib().lq_scaled_mm_noalloc(f, _ptr(A), _ptr(a_scales), _ptr(B), _ptr(b_scales), _ptr(C), M, N, K,
                                    ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_scaled_mm_noalloc", rc)
    return C


def scaled_mm_i32acc(A, a_scales, B, b_scales, C=None, acc=None, variant: Variant | None = None, stream=None):
    """W8A8_INT8 scaled_mm that also returns the exact int32 accumulators."""
    _need(A, "A", (torch.int8,), 2)
    _need(B, "B", (torch.int8,), 2)
    M, N, K = _gemm_operands(W8A8_INT8, A, a_scales, B, b_scales, C)
    if C is None:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=A.device)
    _need(acc, "acc", (torch.int32,), 2, (M, N))
    _one_device(A, acc)
    rc = lib().lq_scaled_mm_i32acc(_ptr(A), _ptr(a_scales), _ptr(B), _ptr(b_scales), _ptr(C), _ptr(acc), M, N, K,
                                   ctypes.byref(variant) if variant is not None else None, _stream(stream))
    _check("lq_scaled_mm_i32acc", rc)
    return C, acc


def quant_per_token(fmt, x: torch.Tensor, q: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                    stream=None):
    """(codes [M, K], scales [M]) of a bf16 [M, K] tensor; e4m3 codes as uint8, int8 codes as int8."""
    f = _fmt(fmt)
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    q, scales = _outputs(x.device, q, (M, K), _code_dtype(f), scales, (M,))
    _one_device(x, q, scales)
    rc = lib().lq_quant_per_token(f, _ptr(x), _ptr(q), _ptr(scales), M, K, _stream(stream))
    _check("lq_quant_per_token", rc)
    return q, scales


def quant_per_token_group128(x: torch.Tensor, q=None, scales=None, stream=None):
    """(e4m3 codes [M, K], scales [M, K/128]) of a bf16 [M, K] tensor."""
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    q, scales = _outputs(x.device, q, (M, K), torch.uint8, scales, (M, max(K // 128, 0)))
    _one_device(x, q, scales)
    rc = lib().lq_quant_per_token_group128(_ptr(x), _ptr(q), _ptr(scales), M, K, _stream(stream))
    _check("lq_quant_per_token_group128", rc)
    return q, scales


def _producer_out(f: int, M: int, K: int, per_block: bool, device, q, scales):
    return _outputs(device, q, (M, K), _code_dtype(f), scales, (M, max(K // 128, 0)) if per_block else (M,))


def _rms_inputs(x, weight, residual):
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    _need(weight, "weight", (torch.bfloat16,), 1, (K,))
    if residual is not None:
        _need(residual, "residual", (torch.bfloat16,), 2, (M, K))
    return M, K


def rms_norm_dynamic_per_token_quant(fmt, x: torch.Tensor, weight: torch.Tensor, eps: float, residual=None,
                                     q=None, scales=None, stream=None):
    """(codes [M, K], scales [M]) of RMSNorm(x [+ residual]) * weight; the
    residual, when given, is overwritten with x + residual."""
    f = _fmt(fmt)
    M, K = _rms_inputs(x, weight, residual)
    q, scales = _producer_out(f, M, K, False, x.device, q, scales)
    _one_device(x, weight, residual, q, scales)
    rc = lib().lq_rms_norm_dynamic_per_token_quant(f, _ptr(x), _ptr(residual) if residual is not None else None,
                                                   _ptr(weight), float(eps), _ptr(q), _ptr(scales), M, K,
                                                   _stream(stream))
    _check("lq_rms_norm_dynamic_per_token_quant", rc)
    return q, scales


def rms_norm_per_block_quant(x: torch.Tensor, weight: torch.Tensor, eps: float, residual=None, q=None,
                             scales=None, stream=None):
    """(e4m3 codes [M, K], scales [M, K/128]) of RMSNorm(x [+ residual]) * weight."""
    M, K = _rms_inputs(x, weight, residual)
    q, scales = _producer_out(FP8_DYNAMIC, M, K, True, x.device, q, scales)
    _one_device(x, weight, residual, q, scales)
    rc = lib().lq_rms_norm_per_block_quant(_ptr(x), _ptr(residual) if residual is not None else None, _ptr(weight),
                                           float(eps), _ptr(q), _ptr(scales), M, K, _stream(stream))
    _check("lq_rms_norm_per_block_quant", rc)
    return q, scales


def _gate_up_width(gate_up) -> tuple[int, int]:
    _need(gate_up, "gate_up", (torch.bfloat16,), 2)
    M, two_i = gate_up.shape
    if two_i % 2:
        raise ValueError("gate_up must have an even number of columns ([g | u])")
    return M, two_i // 2


def silu_and_mul_dynamic_per_token_quant(fmt, gate_up: torch.Tensor, q=None, scales=None, stream=None):
    """(codes [M, I], scales [M]) of silu(gate_up[:, :I]) * gate_up[:, I:]."""
    f = _fmt(fmt)
    M, I = _gate_up_width(gate_up)
    q, scales = _producer_out(f, M, I, False, gate_up.device, q, scales)
    _one_device(gate_up, q, scales)
    rc = lib().lq_silu_and_mul_dynamic_per_token_quant(f, _ptr(gate_up), _ptr(q), _ptr(scales), M, I,
                                                       _stream(stream))
    _check("lq_silu_and_mul_dynamic_per_token_quant", rc)
    return q, scales


def silu_and_mul_per_block_quant(gate_up: torch.Tensor, q=None, scales=None, stream=None):
    """(e4m3 codes [M, I], scales [M, I/128]) of silu(g) * u."""
    M, I = _gate_up_width(gate_up)
    q, scales = _producer_out(FP8_DYNAMIC, M, I, True, gate_up.device, q, scales)
    _one_device(gate_up, q, scales)
    rc = lib().lq_silu_and_mul_per_block_quant(_ptr(gate_up), _ptr(q), _ptr(scales), M, I, _stream(stream))
    _check("lq_silu_and_mul_per_block_quant", rc)
    return q, scales


def quant_per_token_group128_ue8m0(x: torch.Tensor, q=None, scales=None, stream=None):
    """(e4m3 codes [M, K], UE8M0 scale bytes [M, K/128]) of a bf16 [M, K] tensor."""
    _need(x, "x", (torch.bfloat16,), 2)
    M, K = x.shape
    q, scales = _outputs(x.device, q, (M, K), torch.uint8, scales, (M, max(K // 128, 0)), torch.uint8)
    _one_device(x, q, scales)
    rc = lib().lq_quant_per_token_group128_ue8m0(_ptr(x), _ptr(q), _ptr(scales), M, K, _stream(stream))
    _check("lq_quant_per_token_group128_ue8m0", rc)
    return q, scales


def quant_weight_block128_ue8m0(w: torch.Tensor, q=None, scales=None, stream=None):
    """(e4m3 codes [N, K], UE8M0 scale bytes [N/128, K/128]) of a bf16 weight [N, K]."""
    _need(w, "w", (torch.bfloat16,), 2)
    N, K = w.shape
    q, scales = _outputs(w.device, q, (N, K), torch.uint8, scales, (max(N // 128, 0), max(K // 128, 0)),
                         torch.uint8)
    _one_device(w, q, scales)
    rc = lib().lq_quant_weight_block128_ue8m0(_ptr(w), _ptr(q), _ptr(scales), N, K, _stream(stream))
    _check("lq_quant_weight_block128_ue8m0", rc)
    return q, scales


def quant_weight_block128(w: torch.Tensor, q=None, scales=None, stream=None):
    """(e4m3 codes [N, K], scales [N/128, K/128]) of a bf16 weight [N, K]."""
    _need(w, "w", (torch.bfloat16,), 2)
    N, K = w.shape
    q, scales = _outputs(w.device, q, (N, K), torch.uint8, scales, (max(N // 128, 0), max(K // 128, 0)))
    _one_device(w, q, scales)
    rc = lib().lq_quant_weight_block128(_ptr(w), _ptr(q), _ptr(scales), N, K, _stream(stream))
    _check("lq_quant_weight_block128", rc)
    return q, scales


def select_variant(fmt, M: int, N: int, K: int) -> Variant:
    v = Variant()
    _check("lq_select_variant", lib().lq_select_variant(_fmt(fmt), M, N, K, ctypes.byref(v)))
    return v


def load_dispatch_table(path: str | None) -> None:
    _check("lq_load_dispatch_table", lib().lq_load_dispatch_table(None if path is None else path.encode()))


def dispatch_table_size() -> int:
    return int(lib().lq_dispatch_table_size())


def init_device(device: int = 0) -> None:
    _check("lq_init_device", lib().lq_init_device(device))


def reserve_workspace(device: int, nbytes: int) -> None:
    _check("lq_reserve_workspace", lib().lq_reserve_workspace(device, nbytes))


def workspace_bytes(fmt, M, N, K, variant: Variant | None = None) -> int:
    return int(lib().lq_workspace_bytes(_fmt(fmt), M, N, K, ctypes.byref(variant) if variant is not None else None))


def device_status(device: int = 0) -> int:
    """Read and clear the device status word: 0, or LQ_ERR_DEVICE_TIMEOUT (6)."""
    return int(lib().lq_device_status(device))


def set_trace(buf: torch.Tensor | None) -> None:
    """Record 12 globaltimer stamps per CTA of the following scaled_mm launches
    into ``buf`` (a contiguous 1-d int64 CUDA tensor), or stop (None).  The
    library cannot know the grids to come: ``buf`` must hold 12 entries for
    every CTA of the largest launch made while tracing is on."""
    if buf is not None:
        _need(buf, "buf", (torch.int64,), 1)
        _one_device(buf)
    lib().lq_set_trace(None if buf is None else buf.data_ptr())


def declare_static_weights(static: bool = True) -> bool:
    """Declare that weights are never written while a GEMM reading them may
    run, so that a default (None) variant may stream weight tiles before the
    previous kernel finishes; returns the previous setting."""
    return bool(lib().lq_declare_static_weights(1 if static else 0))


def set_fuse_limit(max_slice_bytes: int) -> int:
    """Largest per-CTA activation slice (bytes) for which quant_scaled_mm
    runs one kernel (0 = never, negative = default); returns the old limit."""
    return int(lib().lq_set_fuse_limit(int(max_slice_bytes)))


def test_inject_stall(k_tile: int, wait_limit_ns: int = 0) -> None:
    """Test hook: leave K tile `k_tile` of every CTA unloaded so that a bounded
    wait runs out (-1 = off); `wait_limit_ns` > 0 shortens every wait."""
    _check("lq_test_inject_stall", lib().lq_test_inject_stall(int(k_tile), int(wait_limit_ns)))


def test_silu_bf16(gate: torch.Tensor, stream=None) -> torch.Tensor:
    """Test hook: bf16(silu(gate)) by the producer kernels' own device code."""
    if gate.dtype != torch.bfloat16 or not gate.is_cuda or not gate.is_contiguous():
        raise ValueError("gate must be a contiguous bf16 CUDA tensor")
    out = torch.empty_like(gate)
    _check("lq_test_silu_bf16", lib().lq_test_silu_bf16(_ptr(gate), _ptr(out), gate.numel(), _stream(stream)))
    return out


def status_string(code: int) -> str:
    return lib().lq_status_string(code).decode()


def version() -> str:
    return lib().lq_version().decode()


def call_raw(name: str, *args) -> int:
    """Call a C entry point with raw arguments (for argument-check tests)."""
    return int(getattr(lib(), name)(*args))


@dataclass(frozen=True)
class Problem:
    """A (format, M, N, K) GEMM shape."""
    fmt: int
    M: int
    N: int
    K: int

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def bytes(self) -> int:
        """Algorithmic HBM bytes: weights + activations + scales + bf16 output."""
        if self.fmt in (BLOCK_FP8, BLOCK_FP8_UE8M0):
            per = 1 if self.fmt == BLOCK_FP8_UE8M0 else 4   # UE8M0 scales are bytes
            scales = per * (self.M * (self.K // 128) + (self.N // 128) * (self.K // 128))
        else:
            scales = 4 * (self.M + self.N)
        return self.N * self.K + self.M * self.K + scales + 2 * self.M * self.N
