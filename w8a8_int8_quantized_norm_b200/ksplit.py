"""The row split (split over input channels) of a W8A8 Linear across GPUs.

"SmoothQuant, in depth" -- "Where the scales go in a decoder block": the
o_proj / down_proj style Linears read unsmoothed inputs that are still
quantised per token.  When such a Linear's input channels K are split over
the ranks of a group (rank r holds x[:, K_r] and W[:, K_r]), two things of the
unsplit layer span all slices: the per-token step (max over all K / 127) and
the INT32 accumulator (a sum over all K).  The slices therefore meet twice,
and both meetings are exact:

  1. each rank reduces its slice's row maxima; all-reduce MAX;
  2. each rank quantises its slice with the whole rows' steps and runs the
     INT8 GEMM of its slice to INT32 partial sums; all-reduce SUM (integer
     addition: the unsplit accumulator);
  3. the dequantising epilogue of the summed accumulator.

The weights are quantised the same way once (per-output-channel maxima over
all K by an all-reduce MAX).  Every rank ends with the unsplit layer's
output, bit for bit.  The collectives are torch.distributed all-reduces
(NCCL between GPUs); every arithmetic step runs in libsq.so.

The steps are separate functions so that a caller (or a test) can run the
slices in any order and reduce them itself; ``linear_shard`` and
``quantize_weight_shard`` put the collectives in between.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import sq

Reduce = Callable[[torch.Tensor], None]  # in-place all-reduce of one tensor


class LibOps:
    """The steps of the split on the GPU, through the C ABI."""

    @staticmethod
    def row_absmax(x: torch.Tensor) -> torch.Tensor:
        return sq.row_absmax(x)

    @staticmethod
    def quant_given(x: torch.Tensor, row_absmax: torch.Tensor):
        return sq.quant_per_token_given_absmax(x, row_absmax)

    @staticmethod
    def gemm_i32(Xq: torch.Tensor, Wq: torch.Tensor) -> torch.Tensor:
        return sq.w8a8_gemm_dequant(Xq, Wq, None, None, "i32")

    @staticmethod
    def dequant(acc: torch.Tensor, x_scale: torch.Tensor, w_scale: torch.Tensor,
                epi: str = "bf16") -> torch.Tensor:
        return sq.dequant_i32(acc, x_scale, w_scale, epi)


def torch_reducers(group=None) -> Tuple[Reduce, Reduce]:
    """(all-reduce MAX, all-reduce SUM) over a torch.distributed group."""
    import torch.distributed as dist

    def rmax(t):
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)

    def rsum(t):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)

    return rmax, rsum


# -- the steps ---------------------------------------------------------------

def shard_row_max(x_shard, ops=LibOps):
    """Step 1, local: the slice's max |x| per token (row)."""
    return ops.row_absmax(x_shard)


def shard_partial(x_shard, row_absmax, Wq_shard, ops=LibOps):
    """Step 2, local: codes of the slice with the whole rows' maxima (so the
    step and every code are the unsplit layer's), then the INT32 partial
    accumulator of the slice.  Returns (partial, x_scale)."""
    Xq, x_scale = ops.quant_given(x_shard, row_absmax)
    return ops.gemm_i32(Xq, Wq_shard), x_scale


def finish(acc, x_scale, w_scale, epi: str = "bf16", ops=LibOps):
    """Step 3: the epilogue of the summed accumulator."""
    return ops.dequant(acc, x_scale, w_scale, epi)


# -- with the collectives ------------------------------------------------------

def quantize_weight_shard(W_shard, reduce_max: Optional[Reduce] = None, ops=LibOps):
    """INT8 codes of this rank's slice W[:, K_r] and the per-output-channel
    scales of the whole W (max over all K / 127).  Returns (Wq_shard, w_scale)."""
    if reduce_max is None:
        reduce_max, _ = torch_reducers()
    am = ops.row_absmax(W_shard)
    reduce_max(am)
    return ops.quant_given(W_shard, am)


def linear_shard(x_shard, Wq_shard, w_scale, epi: str = "bf16",
                 reduce_max: Optional[Reduce] = None, reduce_sum: Optional[Reduce] = None,
                 ops=LibOps):
    """The split Linear on this rank's slice: every rank returns the whole
    layer's output [M, N]."""
    if reduce_max is None or reduce_sum is None:
        rmax, rsum = torch_reducers()
        reduce_max = reduce_max or rmax
        reduce_sum = reduce_sum or rsum
    am = shard_row_max(x_shard, ops)
    reduce_max(am)
    acc, x_scale = shard_partial(x_shard, am, Wq_shard, ops)
    reduce_sum(acc)
    return finish(acc, x_scale, w_scale, epi, ops)
