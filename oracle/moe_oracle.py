"""Plain CPU oracle for the grouped (mixture-of-experts) quantized GEMM.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU legs may import or run this module.  The library under
``quantized_linear_gemm_b200/`` never calls it, links it or shares code with it.

Where it comes from
-------------------
The ai-radar.it page "Helion in vLLM: il tuning dei GEMM diventa ricerca, non
artigianato GPU", section "Oltre Hopper: Blackwell, AMD, TPU e il perimetro
del fork", names the MoE backend as the next target: many experts of small
size, where the Split-K and Swap-AB choices matter more.  It gives no
interface.  The plainest reading, used here: every expert is an ordinary
quantized linear layer (FP8_Dynamic or W8A8_INT8, the formats of
``lq_oracle``), and the tokens routed to expert e form a contiguous block of
rows:

* A [T, K] activation codes, tokens sorted by expert: rows
  offsets[e] .. offsets[e+1]-1 go to expert e (offsets[0] = 0,
  offsets[E] = T, non-decreasing); a_scales [T] per token;
* B [E, N, K] weight codes, b_scales [E, N] per output channel;
* C [T, N], row t = scaled_mm of token t with its expert's weights.
"""

from __future__ import annotations

import numpy as np

from oracle import lq_oracle as O


def check_offsets(offsets, T: int, E: int) -> np.ndarray:
    """The expert offsets [E + 1] as int64: expert e's tokens are the rows
    [offsets[e], offsets[e + 1]) of A, so the table starts at 0, never
    decreases and ends at T (anything else is refused).

    Source: the routing table of the grouped GEMM (MoE is named as the next
    target by ai-radar.it, section "Oltre Hopper: Blackwell, AMD, TPU e il
    perimetro del fork"; the layout is this oracle's reading).
    """
    off = np.asarray(offsets, dtype=np.int64)
    if off.shape != (E + 1,) or off[0] != 0 or off[-1] != T or np.any(np.diff(off) < 0):
        raise ValueError("offsets must be non-decreasing, start at 0 and end at T")
    return off


def grouped_scaled_mm_ref(fmt: str, a_codes, a_scales, b_codes, b_scales, offsets) -> np.ndarray:
    """C [T, N] (float64, exact product rounded once per lq_oracle's
    definition) of the grouped quantized GEMM."""
    a_codes = np.asarray(a_codes)
    b_codes = np.asarray(b_codes)
    T, K = a_codes.shape
    E, N, K2 = b_codes.shape
    assert K == K2
    off = check_offsets(offsets, T, E)
    a_scales = np.asarray(a_scales, dtype=np.float32)
    b_scales = np.asarray(b_scales, dtype=np.float32).reshape(E, N)
    C = np.zeros((T, N), dtype=np.float64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            C[lo:hi] = O.scaled_mm_ref(fmt, a_codes[lo:hi], a_scales[lo:hi], b_codes[e], b_scales[e])
    return C

