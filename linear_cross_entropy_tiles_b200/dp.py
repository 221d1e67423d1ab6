"""Data-parallel FLCE: one process per GPU, each holding its own rows.

A training step over a global batch split by rows across ranks (the same W
on every rank) needs two exchanges around the per-rank kernels:

  1. before any G is formed: the number of non-ignored labels over all
     ranks, the divisor of the global mean loss (torchtune issue #1228's
     recipe averages the loss over the batch before backward);
  2. after backward: the sum over ranks of every rank's dW = G_r^T X_r, and
     the sum of the ranks' loss shares.  dW is summed in fp32 by default:
     each rank writes its share in fp32 (the library's dw_fp32 output, the
     same fp32 sums it would otherwise round to bf16), so the cross-rank sum
     adds no rounding beyond fp32's; summing bf16 shares in bf16 instead
     rounds every partial sum to 8 bits, an error that grows with the number
     of ranks.

dX needs no exchange: a rank's rows of dX depend only on its rows.  The
collectives go through torch.distributed (NCCL on GPUs); all arithmetic
runs in the library's kernels (flce_count_valid, flce_fused_global).
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

from . import binding


def data_parallel_step(count_local: Callable[[], torch.Tensor],
                       compute: Callable[[torch.Tensor], tuple],
                       group=None, reduce_dw: bool = True):
    """The exchange pattern of a data-parallel FLCE step.

    count_local() returns this rank's count of non-ignored labels as an int64
    [1] tensor; compute(n_global) returns (loss share, dX, dW) for this rank
    with the mean taken over n_global rows.  Returns (global mean loss, this
    rank's dX, dW summed over ranks, n_global).  Every rank must call it the
    same number of times, in the same order.
    """
    n = count_local()
    dist.all_reduce(n, op=dist.ReduceOp.SUM, group=group)
    loss, dX, dW = compute(n)
    dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    if reduce_dw:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM, group=group)
    return loss, dX, dW, n


def fused_dp(X: torch.Tensor, W: torch.Tensor, labels: torch.Tensor, group=None,
             ignore_index: int = -100, softcap: float = 0.0, dloss: float = 1.0,
             ws: torch.Tensor | None = None, reduce_dw: bool = True, shift_seq_len: int = 0,
             dw_fp32: bool = True):
    """Forward and backward of FLCE over the rows of all ranks in `group`.

    X [BT_r, H] and labels [BT_r] are this rank's rows (whole sequences when
    shift_seq_len > 0, as in binding.fused); W [V, H] is the same on every
    rank.  Returns (loss [1]: the mean over all ranks' non-ignored rows, dX:
    this rank's rows, dW: summed over ranks unless reduce_dw is False,
    n_global [1] int64).  With dw_fp32 (the default) dW is fp32, written in
    fp32 by each rank and summed in fp32; otherwise it has X's dtype and the
    collective sums it in that dtype.
    """
    return data_parallel_step(
        lambda: binding.count_valid(X, W, labels, ignore_index, shift_seq_len=shift_seq_len),
        lambda n: binding.fused(X, W, labels, ignore_index=ignore_index, softcap=softcap,
                                dloss=dloss, ws=ws, n_valid_global=n,
                                shift_seq_len=shift_seq_len, dw_fp32=dw_fp32),
        group=group, reduce_dw=reduce_dw)
