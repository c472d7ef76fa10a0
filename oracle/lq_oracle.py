"""Plain CPU oracle for the quantized linear-layer GEMM (``scaled_mm``) and its
activation / weight quantizers.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or
run this module.  The library under ``quantized_linear_gemm_b200/`` never
calls it, links it or shares code with it.

What is computed, and where it is defined
-----------------------------------------
Source pages: "Building a High-Performance and Portable vLLM Linear Backend
with Helion" (PyTorch blog; section "Helion Linear Backend > Scope") defines
the three formats:

* FP8_Dynamic - FP8 activations with one scale per token, FP8 weights with one
  scale per output channel;
* W8A8_INT8   - the same scale granularity with INT8 codes;
* Block_FP8   - FP8 with one activation scale per 1x128 group and one weight
  scale per 128x128 block.

The same page, section "Kernel Implementation", and the techfeed.io summary of
it (section "何が面白いのか") define the
Split-K and Swap-AB variants as rewrites of the *same* product, so the oracle
has one definition of C and only uses split / transposed loop orders as
self-checks (``acc_split_k``, ``acc_swap_ab``).

The blog and its re-reports leave the numeric details open.  Readings adopted here (each listed
in the design notes of the repository):

* FP8 means OCP e4m3fn (finite max 448, no infinities, NaN = S.1111.111).
* Encoding to e4m3 rounds to nearest, ties to even, and saturates to +-448.
* INT8 encoding is symmetric: clamp(round_half_even(v), -127, 127).
* A quantization scale is s = max(fp32(amax / Q), 2^-126) with Q = 448 (e4m3)
  or 127 (int8), amax the largest magnitude over the scale's group, and the
  code is enc(fp32(x / s)) with a correctly rounded fp32 division.
* Weights are stored [N, K] (output channel major, K contiguous); the code
  sample of the techfeed.io summary (section "何が面白いのか") indexes the
  logical operand as b[k, n].
* Output C is the exact product rounded once; the oracle returns it in fp64.

Exactness.  Every finite e4m3 value is an integer multiple of 2^-9 whose
magnitude times 2^9 is at most 229376 < 2^18, so a product of two codes is an
integer times 2^-18 below 2^36 in magnitude, and a sum over K <= 25600 < 2^15
terms stays below 2^51: the accumulator is computed exactly in int64.  INT8
products are below 2^14 and sums over K <= 25600 stay below 2^29 < 2^31.
Scales are then applied in fp64.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
INT8_QMAX = 127.0
FP32_MIN_NORMAL = np.float32(2.0 ** -126)
BLOCK = 128  # group / block edge of Block_FP8

FMT_FP8_DYNAMIC = "fp8_dynamic"
FMT_W8A8_INT8 = "w8a8_int8"
FMT_BLOCK_FP8 = "block_fp8"
FORMATS = (FMT_FP8_DYNAMIC, FMT_W8A8_INT8, FMT_BLOCK_FP8)


# ---------------------------------------------------------------------------
# e4m3fn codec (format reading: OCP 8-bit float, E4M3 "fn" variant)
# ---------------------------------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each e4m3fn byte, as float64 (NaN for S.1111.111).

    exponent field e (4 bits), mantissa field m (3 bits):
    e == 0 -> (-1)^s * m * 2^-9 ; otherwise (-1)^s * (8 + m) * 2^(e - 10).

    Source: "FP8" of the PyTorch blog "Building a High-Performance and Portable vLLM Linear Backend
    with Helion", section "Helion Linear Backend > Scope", read as the OCP FP8 E4M3 ("fn") format.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.ldexp(1.0, (e - 10)))
    val = np.where(s == 1, -mag, mag)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return val.astype(np.float64)


def e4m3_decode_int(codes) -> np.ndarray:
    """e4m3fn value times 2^9, as an exact int64 (NaN codes are rejected).

    Source: as e4m3_decode; the integer form makes the accumulation below exact.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    if np.any((e == 15) & (m == 7)):
        raise ValueError("NaN e4m3 code in an operand")
    # normal: (8+m) * 2^(e-10) * 2^9 = (8+m) << (e-1)   (e >= 1)
    mag = np.where(e == 0, m, (8 + m) << np.maximum(e - 1, 0))
    return np.where(s == 1, -mag, mag).astype(np.int64)


def e4m3_encode(v) -> np.ndarray:
    """Round fp32 values to e4m3fn: nearest, ties to even, saturating at +-448.

    Works in float64, where every fp32 input and every scaling by a power of
    two below is exact.  The sign of the input is kept (so -0.0 and negative
    values that round to zero give 0x80).

    Source: "FP8" of the PyTorch blog "Building a High-Performance and Portable vLLM Linear Backend
    with Helion", section "Helion Linear Backend > Scope"; the rounding (nearest even, saturating) is
    this oracle's reading.
    """
    x = np.asarray(v, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value given to the e4m3 encoder")
    a = np.abs(x.astype(np.float64))
    sign = np.signbit(x).astype(np.int64)
    _, ex = np.frexp(a)                     # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)              # binade exponent; subnormal range below 2^-6
    quantum = np.ldexp(1.0, e - 3)          # 3 mantissa bits
    mag = np.rint(a / quantum) * quantum    # rint: round half to even
    mag = np.minimum(mag, E4M3_MAX)         # saturate to the largest finite value
    sub = mag < 2.0 ** -6
    _, ex2 = np.frexp(np.where(sub, 1.0, mag))
    E = ex2 - 1
    mant_norm = np.rint(np.where(sub, 0.0, mag / np.ldexp(1.0, E) * 8.0 - 8.0)).astype(np.int64)
    code_norm = ((E + 7) << 3) | mant_norm
    code_sub = np.rint(mag / 2.0 ** -9).astype(np.int64)
    code = np.where(sub, code_sub, code_norm) | (sign << 7)
    return code.astype(np.uint8)


def int8_encode(v) -> np.ndarray:
    """Symmetric int8 code: clamp(round_half_even(v), -127, 127).

    Source: W8A8_INT8 of the PyTorch blog "Building a High-Performance and Portable vLLM Linear Backend
    with Helion", section "Helion Linear Backend > Scope"; the symmetric half-even code is this
    oracle's reading.
    """
    x = np.asarray(v, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite value given to the int8 encoder")
    return np.clip(np.rint(x.astype(np.float64)), -INT8_QMAX, INT8_QMAX).astype(np.int8)


# ---------------------------------------------------------------------------
# Quantizers (formats from the blog's "Scope" section; rule as read above)
# ---------------------------------------------------------------------------

def _qmax(fmt: str) -> float:
    return INT8_QMAX if fmt == FMT_W8A8_INT8 else E4M3_MAX


def _encode(fmt: str, y) -> np.ndarray:
    return int8_encode(y) if fmt == FMT_W8A8_INT8 else e4m3_encode(y)


def scale_from_amax(amax, qmax: float) -> np.ndarray:
    """s = max(fp32(amax / qmax), 2^-126), one correctly rounded fp32 division.

    Source: the per-token / per-channel / per-group scales of the PyTorch blog "Building a
    High-Performance and Portable vLLM Linear Backend with Helion", section "Helion Linear Backend >
    Scope"; the division and the 2^-126 floor are this oracle's reading.
    """
    a = np.asarray(amax, dtype=np.float32)
    s = a / np.float32(qmax)
    return np.maximum(s, FP32_MIN_NORMAL).astype(np.float32)


def quantize_groups(x, fmt: str, axis_len: int):
    """Quantize each contiguous group of ``axis_len`` values along the last axis.

    x: float32 array [..., L] with L % axis_len == 0.
    Returns (codes [..., L], scales [..., L // axis_len] float32).

    Source: the step shared by the three scale granularities of the PyTorch blog "Building a
    High-Performance and Portable vLLM Linear Backend with Helion", section "Helion Linear Backend >
    Scope".
    """
    x = np.asarray(x, dtype=np.float32)
    L = x.shape[-1]
    if L % axis_len:
        raise ValueError("row length is not a multiple of the group length")
    g = x.reshape(x.shape[:-1] + (L // axis_len, axis_len))
    amax = np.max(np.abs(g), axis=-1)
    s = scale_from_amax(amax, _qmax(fmt))
    y = g / s[..., None]                  # float32 / float32: IEEE round to nearest
    codes = _encode(fmt, y.astype(np.float32))
    return codes.reshape(x.shape), s


def quant_per_token(x, fmt: str):
    """Dynamic per-token activation quantization (FP8_Dynamic, W8A8_INT8).

    x: [M, K] values of the bf16 activations (as float32).  One scale per row.
    The blog lists this step as ``dynamic_per_token_scaled_fp8_quant`` among
    the kernels it integrates (24-ai.news report, section "kernels integrated
    into vLLM").
    """
    x = np.asarray(x, dtype=np.float32)
    codes, s = quantize_groups(x, fmt, x.shape[-1])
    return codes, s.reshape(x.shape[0])


def quant_per_channel(w, fmt: str):
    """Per-output-channel weight quantization of W stored [N, K]: one scale per n.

    Source: FP8_Dynamic / W8A8_INT8 weights, one scale per output channel (PyTorch blog "Building a
    High-Performance and Portable vLLM Linear Backend with Helion", section "Helion Linear Backend >
    Scope").
    """
    return quant_per_token(w, fmt)


def quant_per_token_group128(x):
    """1x128 group activation quantization of Block_FP8 (``per_token_group_fp8_quant``).

    x: [M, K], K % 128 == 0.  Returns (codes [M, K], scales [M, K/128]).

    Source: Block_FP8 activations (PyTorch blog "Building a High-Performance and Portable vLLM Linear
    Backend with Helion", section "Helion Linear Backend > Scope"); the kernel is named in the
    24-ai.news report, section "vLLMに統合されたカーネル".
    """
    return quantize_groups(np.asarray(x, dtype=np.float32), FMT_BLOCK_FP8, BLOCK)


def quant_weight_block128(w):
    """128x128 block weight quantization of Block_FP8 for W stored [N, K].

    One scale per (n-block, k-block) from the amax over the whole block.
    Returns (codes [N, K] uint8, scales [N/128, K/128] float32).

    Source: Block_FP8 weights, one scale per 128 x 128 block (PyTorch blog "Building a High-Performance
    and Portable vLLM Linear Backend with Helion", section "Helion Linear Backend > Scope").
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    if N % BLOCK or K % BLOCK:
        raise ValueError("Block_FP8 weights need N and K multiples of 128")
    NB, KB = N // BLOCK, K // BLOCK
    blocks = w.reshape(NB, BLOCK, KB, BLOCK)
    amax = np.max(np.abs(blocks), axis=(1, 3))                 # [NB, KB]
    s = scale_from_amax(amax, E4M3_MAX)
    y = blocks / s[:, None, :, None]
    codes = e4m3_encode(y.astype(np.float32)).reshape(N, K)
    return codes, s


# ---------------------------------------------------------------------------
# Exact accumulators and the reference product
# ---------------------------------------------------------------------------

def operand_int(fmt: str, codes) -> np.ndarray:
    """Operand codes as exact int64: e4m3 value * 2^9, or the int8 value.

    Source: the operands of the PyTorch blog "Building a High-Performance and Portable vLLM Linear
    Backend with Helion", section "Helion Linear Backend > Scope" in the exact integer form acc_exact
    sums.
    """
    if fmt == FMT_W8A8_INT8:
        return np.asarray(codes, dtype=np.int8).astype(np.int64)
    return e4m3_decode_int(codes)


def acc_exact(fmt: str, a_codes, b_codes) -> np.ndarray:
    """acc[m, n] = sum_k A[m, k] * B[n, k] in int64 (e4m3 operands in 2^-9 units).

    This is the tiled loop of the blog's unified kernel (``acc = dot(a[tile_m,
    tile_k], b[tile_k, tile_n], acc)``) with the tiling removed: the full K sum.
    """
    A = operand_int(fmt, a_codes)
    B = operand_int(fmt, b_codes)
    return A @ B.T          # numpy int64 matmul: exact, no BLAS


def acc_exact_blocks(a_codes, b_codes) -> list:
    """Per-128-K-block exact e4m3 accumulators (list over kb of int64 [M, N]).

    Source: Block_FP8's per-128-K partial products (PyTorch blog "Building a High-Performance and
    Portable vLLM Linear Backend with Helion", section "Helion Linear Backend > Scope").
    """
    A = e4m3_decode_int(a_codes)
    B = e4m3_decode_int(b_codes)
    K = A.shape[1]
    return [A[:, kb:kb + BLOCK] @ B[:, kb:kb + BLOCK].T for kb in range(0, K, BLOCK)]


def scaled_mm_ref(fmt: str, a_codes, a_scales, b_codes, b_scales) -> np.ndarray:
    """Reference C[m, n] in fp64 for FP8_Dynamic and W8A8_INT8.

    C = acc * unit * a_s[m] * b_s[n], unit = 2^-18 for e4m3 and 1 for int8
    (per-token activation scale times per-channel weight scale, blog "Scope").
    """
    if fmt == FMT_BLOCK_FP8:
        return blockwise_ref(a_codes, a_scales, b_codes, b_scales)
    acc = acc_exact(fmt, a_codes, b_codes).astype(np.float64)
    unit = 1.0 if fmt == FMT_W8A8_INT8 else 2.0 ** -18
    a_s = np.asarray(a_scales, dtype=np.float32).astype(np.float64)
    b_s = np.asarray(b_scales, dtype=np.float32).astype(np.float64)
    return acc * unit * a_s[:, None] * b_s[None, :]


def blockwise_ref(a_codes, a_scales, b_codes, b_scales) -> np.ndarray:
    """Reference C for Block_FP8 in fp64.

    C[m, n] = sum_kb acc_kb[m, n] * 2^-18 * a_s[m, kb] * b_s[n // 128, kb]
    (1x128 activation scales times 128x128 weight scales, blog "Scope").
    """
    a_s = np.asarray(a_scales, dtype=np.float32).astype(np.float64)   # [M, KB]
    b_s = np.asarray(b_scales, dtype=np.float32).astype(np.float64)   # [NB, KB]
    blocks = acc_exact_blocks(a_codes, b_codes)
    M, N = blocks[0].shape
    nb_of_n = np.arange(N) // BLOCK
    C = np.zeros((M, N), dtype=np.float64)
    for kb, acc in enumerate(blocks):
        C += acc.astype(np.float64) * 2.0 ** -18 * a_s[:, kb][:, None] * b_s[nb_of_n, kb][None, :]
    return C


# ---------------------------------------------------------------------------
# Variant loop orders, used only as self-checks of the single definition
# ---------------------------------------------------------------------------

def split_ranges(num_k_tiles: int, split_k: int):
    """K-tile range of each split s: [floor(s*T/S), floor((s+1)*T/S)).

    Reading of the blog's Split-K ("partitions the K dimension across multiple
    thread blocks"): an even floor partition of the 128-wide K tiles; splits
    may be empty when S > T.
    """
    T, S = num_k_tiles, split_k
    return [((s * T) // S, ((s + 1) * T) // S) for s in range(S)]


def acc_split_k(fmt: str, a_codes, b_codes, split_k: int) -> np.ndarray:
    """Split-K order: one exact partial per K range, summed in order s = 0..S-1.

    Source: the Split-K variant (PyTorch blog "Building a High-Performance and Portable vLLM Linear
    Backend with Helion", section "Kernel Implementation"); a self-check, not a second definition.
    """
    A = operand_int(fmt, a_codes)
    B = operand_int(fmt, b_codes)
    K = A.shape[1]
    T = -(-K // BLOCK)
    total = np.zeros((A.shape[0], B.shape[0]), dtype=np.int64)
    for lo, hi in split_ranges(T, split_k):
        k0, k1 = lo * BLOCK, min(hi * BLOCK, K)
        if k1 > k0:
            total = total + A[:, k0:k1] @ B[:, k0:k1].T
    return total


def acc_swap_ab(fmt: str, a_codes, b_codes) -> np.ndarray:
    """Swap-AB order: compute (B^T A^T)^T, i.e. the product with roles exchanged.

    The accumulator is built as D[n, m] = sum_k B[n, k] * A[m, k] by an explicit
    loop over K (not via ``acc_exact``) and transposed at the end.

    Source: the Swap-AB variant (PyTorch blog "Building a High-Performance and Portable vLLM Linear
    Backend with Helion", section "Kernel Implementation"; its formula is garbled in the extracted text
    and read as (B^T A^T)^T).
    """
    A = operand_int(fmt, a_codes)
    B = operand_int(fmt, b_codes)
    D = np.zeros((B.shape[0], A.shape[0]), dtype=np.int64)
    for k in range(A.shape[1]):
        D += np.outer(B[:, k], A[:, k])
    return D.T


# ---------------------------------------------------------------------------
# Acceptance
# ---------------------------------------------------------------------------

def bf16_tolerance(C_ref) -> np.ndarray:
    """Per-element bound 2^-7 * |C_ref| + 1e-3 * rms(C_ref) for a bf16 result.

    Source: none in the blog or its re-reports; the acceptance bound adopted for bf16 outputs.
    """
    C_ref = np.asarray(C_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(C_ref * C_ref))) if C_ref.size else 0.0
    return 2.0 ** -7 * np.abs(C_ref) + 1e-3 * rms


def within_tolerance(C, C_ref, rms_of=None):
    """(ok, worst ratio |C - C_ref| / bound).  ``rms_of`` overrides the rms source
    (the full reference when C_ref is only a sample of it).

    Source: as bf16_tolerance.
    """
    C = np.asarray(C, dtype=np.float64)
    C_ref = np.asarray(C_ref, dtype=np.float64)
    src = C_ref if rms_of is None else np.asarray(rms_of, dtype=np.float64)
    rms = float(np.sqrt(np.mean(src * src))) if src.size else 0.0
    bound = 2.0 ** -7 * np.abs(C_ref) + 1e-3 * rms
    err = np.abs(C - C_ref)
    if err.size == 0:
        return True, 0.0
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / np.where(bound > 0, bound, 1.0), np.where(err > 0, np.inf, 0.0))
    worst = float(np.max(ratio))
    return bool(np.all(err <= bound)), worst
