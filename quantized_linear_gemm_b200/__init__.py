"""lq: quantized linear-layer GEMM (scaled_mm) for B200 (sm_100a).

The compute path is the C-ABI library ``liblq.so`` built from ``csrc/``;
this package only marshals arguments to it (see ``lq.py``).  Importing the
package does not load the library; the first call does, and fails loudly if
it is missing.
"""

__all__ = ["lq", "inputs"]
