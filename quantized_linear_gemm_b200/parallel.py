"""N-sliced (column-parallel) quantized linear over several GPUs.

Each rank holds a contiguous slice of the output channels of the weight
(rows [n0, n1) of B [N, K], with their scales and bias); the activations are
replicated.  The slices need no exchange to compute: every rank runs
``lq_scaled_mm`` (or ``lq_scaled_mm_bias``) on its own slice, and the slices
of C are gathered over NCCL only when the caller wants the full [M, N]
output (a following row-parallel layer would consume the slice as it is).

Slices are equal and aligned: N must split into ``world`` parts that are
multiples of ``align`` (8 for FP8_Dynamic / W8A8_INT8, 128 for the Block_FP8
formats, whose weight scales cover 128 output channels).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from quantized_linear_gemm_b200 import lq


def shard_bounds(N: int, world: int, rank: int, align: int) -> tuple[int, int]:
    """[n0, n1) of rank `rank` out of `world` equal slices of N output
    channels, each a multiple of `align`."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    if N % (world * align):
        raise ValueError(f"N = {N} does not split into {world} slices of a multiple of {align}")
    part = N // world
    return rank * part, (rank + 1) * part


def _align(fmt) -> int:
    return 128 if lq._fmt(fmt) in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0) else 8


@dataclass
class ColumnParallelLinear:
    """The slice of a quantized linear layer held by one rank."""
    fmt: object
    B: torch.Tensor          # [N / world, K] codes of this rank's output channels
    b_scales: torch.Tensor   # their scales ([N / world] or [N / world / 128, K / 128])
    bias: torch.Tensor | None
    n0: int
    n1: int
    N: int

    @classmethod
    def from_full(cls, fmt, B, b_scales, bias=None, rank: int = 0, world: int = 1):
        """Take this rank's slice of a full weight (codes [N, K], scales, bias [N])."""
        N = B.shape[0]
        n0, n1 = shard_bounds(N, world, rank, _align(fmt))
        if lq._fmt(fmt) in (lq.BLOCK_FP8, lq.BLOCK_FP8_UE8M0):
            sb = b_scales[n0 // 128:n1 // 128]
        else:
            sb = b_scales[n0:n1]
        return cls(fmt, B[n0:n1].contiguous(), sb.contiguous(),
                   None if bias is None else bias[n0:n1].contiguous(), n0, n1, N)

    def forward_local(self, A, a_scales, stream=None, gemm=None, gemm_bias=None) -> torch.Tensor:
        """C[:, n0:n1] of this rank, [M, N / world] bf16."""
        if self.bias is None:
            return (gemm or lq.scaled_mm)(self.fmt, A, a_scales, self.B, self.b_scales, stream=stream)
        return (gemm_bias or lq.scaled_mm_bias)(self.fmt, A, a_scales, self.B, self.b_scales, self.bias,
                                                stream=stream)

    def forward(self, A, a_scales, group=None, gather: bool = True, stream=None, gemm=None, gemm_bias=None):
        """This rank's slice, or (gather=True) the full C [M, N] on every rank,
        gathered with one all-gather of the slices."""
        C_local = self.forward_local(A, a_scales, stream=stream, gemm=gemm, gemm_bias=gemm_bias)
        if not gather:
            return C_local
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        if world == 1:
            return C_local
        parts = [torch.empty_like(C_local) for _ in range(world)]
        dist.all_gather(parts, C_local.contiguous(), group=group)
        return torch.cat(parts, dim=1)
