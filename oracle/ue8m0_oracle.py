"""Plain CPU oracle for Block_FP8 with UE8M0 (power-of-two) scales.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs may import or run this module.  The library under
``quantized_linear_gemm_b200/`` never calls it, links it or shares code with it.

Where it comes from
-------------------
The 24-ai.news report "HelionがvLLMに統合：PyTorchネイティブDSLがCUDAカーネルを
代替し、Qwen3モデルのFP8推論を高速化", section "実際の制限事項", notes that the
per-group quantization kernel is not yet compatible with the UE8M0 scale format
that DeepGEMM requires on B200.  The report does not define UE8M0.  Reading used
here (the OCP microscaling E8M0 scale type): an unsigned byte b holding a
power of two, value 2^(b - 127) for b in 0..254 (255 is NaN and never
produced).  A UE8M0 scale is the smallest power of two s with amax / s <= Q
(Q = 448 for e4m3), so no code saturates:

    e = ceil(log2(amax / 448)), clamped to [-127, 127];  s = 2^e;
    q = enc_e4m3(x / s)     (x / s is exact: s is a power of two);
    byte = e + 127.

An all-zero group gets e = -127 (byte 0).  Groups are those of Block_FP8: 1 x 128
for activations, 128 x 128 for weights; the product is ``lq_oracle.blockwise_ref``
with the decoded scales.
"""

from __future__ import annotations

import numpy as np

from oracle import lq_oracle as O

E8M0_BIAS = 127


def e8m0_decode(b) -> np.ndarray:
    """Scale bytes -> float64 values 2^(b - 127) (255 -> NaN).

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    b = np.asarray(b, dtype=np.int64)
    v = np.exp2((b - E8M0_BIAS).astype(np.float64))
    return np.where(b == 255, np.nan, v)


def ue8m0_exponent(amax) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2^e, clamped to [-127, 127];
    amax = 0 gives -127.  Exact: 448 = 7 * 2^6, so the test is
    amax * 2^-e <= 448 decided on the float64 significand and exponent.

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    a = np.asarray(amax, dtype=np.float64)
    m, ex = np.frexp(a)                 # a = m * 2^ex, m in [0.5, 1)
    # 448 * 2^e = 0.875 * 2^(e + 9): amax <= it  <=>  ex < e + 9, or ex == e + 9 and m <= 0.875
    e = np.where(m <= 0.875, ex - 9, ex - 8)
    e = np.where(a == 0, -127, e)
    return np.clip(e, -127, 127).astype(np.int64)


def quantize_groups_ue8m0(x, axis_len: int):
    """Codes [..., L] and scale bytes [..., L / axis_len] of contiguous groups.

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    x = np.asarray(x, dtype=np.float32)
    L = x.shape[-1]
    if L % axis_len:
        raise ValueError("row length is not a multiple of the group length")
    g = x.reshape(x.shape[:-1] + (L // axis_len, axis_len)).astype(np.float64)
    e = ue8m0_exponent(np.max(np.abs(g), axis=-1))
    y = g * np.exp2(-e.astype(np.float64))[..., None]      # exact scaling by a power of two
    codes = O.e4m3_encode(y).reshape(x.shape)
    return codes, (e + E8M0_BIAS).astype(np.uint8)


def quant_per_token_group128_ue8m0(x):
    """1 x 128 activation groups: (codes [M, K], scale bytes [M, K/128]).

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    return quantize_groups_ue8m0(x, O.BLOCK)


def quant_weight_block128_ue8m0(w):
    """128 x 128 weight blocks of W [N, K]: (codes [N, K], scale bytes [N/128, K/128]).

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    if N % O.BLOCK or K % O.BLOCK:
        raise ValueError("Block_FP8 weights need N and K multiples of 128")
    NB, KB = N // O.BLOCK, K // O.BLOCK
    blocks = w.reshape(NB, O.BLOCK, KB, O.BLOCK).astype(np.float64)
    e = ue8m0_exponent(np.max(np.abs(blocks), axis=(1, 3)))      # [NB, KB]
    y = blocks * np.exp2(-e.astype(np.float64))[:, None, :, None]
    codes = O.e4m3_encode(y).reshape(N, K)
    return codes, (e + E8M0_BIAS).astype(np.uint8)


def blockwise_ue8m0_ref(a_codes, a_bytes, b_codes, b_bytes) -> np.ndarray:
    """C [M, N] in fp64: the Block_FP8 product with the decoded power-of-two scales.

    Source: 24-ai.news report, section "実際の制限事項" (UE8M0 scales on B200), read as the OCP microscaling
    E8M0 scale.
    """
    return O.blockwise_ref(a_codes, e8m0_decode(a_bytes), b_codes, e8m0_decode(b_bytes))
