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
runs in the library's kernels (flce_count_valid, flce_fused_global,
flce_fused_global_sliced).

The dW reduction can overlap the end of the computation: with dw_slices,
the library hands dW over in vocabulary slices (a CUDA event per slice, the
last row chunk's dW GEMM run slice by slice), and a side stream reduces each
finished slice while the next one is computed.  It is an all-reduce per
slice (every rank gets the whole summed dW, as plain data parallelism
wants), or with dw_shard a reduction of slice r onto rank r (a reduce-
scatter: rank r keeps rows [a_r, b_r) of the summed dW, the FSDP layout of
torchtune issue #1228's distributed recipes).
"""
from __future__ import annotations

import contextlib
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


def data_parallel_step_sliced(count_local: Callable[[], torch.Tensor],
                              compute: Callable[[torch.Tensor, list], tuple],
                              bounds: list, group=None, shard: bool = False):
    """data_parallel_step with dW reduced slice by slice as it becomes final.

    bounds: [(a_s, b_s)] row ranges of dW (the same on every rank; with
    shard, one per rank).  compute(n_global, events) returns (loss share,
    dX, dW) having recorded events[s] (torch.cuda.Event) once rows
    [a_s, b_s) of dW are final; events is None for CPU tensors, which are
    final when compute returns.  Each slice is all-reduced, or with shard
    reduced onto rank s, on a side stream that waits for its event, so the
    reduction of one slice overlaps the computation of the next.  Returns
    (global mean loss, dX, dW, n_global): dW the whole summed [V, H] tensor,
    or with shard this rank's rows [a_rank, b_rank) of it.
    """
    world = dist.get_world_size(group)
    if shard and len(bounds) != world:
        raise ValueError("a sharded dW needs one slice per rank")
    n = count_local()
    dist.all_reduce(n, op=dist.ReduceOp.SUM, group=group)
    on_gpu = n.is_cuda
    events = [torch.cuda.Event() for _ in bounds] if on_gpu else None
    loss, dX, dW = compute(n, events)
    side = _side_stream(dW.device) if on_gpu else None
    works = []
    with (torch.cuda.stream(side) if on_gpu else contextlib.nullcontext()):
        for s, (a, b) in enumerate(bounds):
            if on_gpu:
                side.wait_event(events[s])
            if b <= a:
                continue
            if shard:
                dst = dist.get_global_rank(group, s) if group is not None else s
                works.append(dist.reduce(dW[a:b], dst=dst, op=dist.ReduceOp.SUM, group=group,
                                         async_op=True))
            else:
                works.append(dist.all_reduce(dW[a:b], op=dist.ReduceOp.SUM, group=group,
                                             async_op=True))
    dist.all_reduce(loss, op=dist.ReduceOp.SUM, group=group)
    for w in works:
        w.wait()  # on a GPU: the current stream waits for the reductions
    if shard:
        a, b = bounds[dist.get_rank(group)]
        dW = dW[a:b]
    return loss, dX, dW, n


_SIDE = {}


def _side_stream(device) -> torch.cuda.Stream:
    """One side stream per device for the slice reductions."""
    key = torch.device(device).index
    if key not in _SIDE:
        _SIDE[key] = torch.cuda.Stream(device=device)
    return _SIDE[key]


def fused_dp(X: torch.Tensor, W: torch.Tensor, labels: torch.Tensor, group=None,
             ignore_index: int = -100, softcap: float = 0.0, dloss: float = 1.0,
             ws: torch.Tensor | None = None, reduce_dw: bool = True, shift_seq_len: int = 0,
             dw_fp32: bool = True, dw_slices: int = 0, dw_shard: bool = False):
    """Forward and backward of FLCE over the rows of all ranks in `group`.

    X [BT_r, H] and labels [BT_r] are this rank's rows (whole sequences when
    shift_seq_len > 0, as in binding.fused); W [V, H] is the same on every
    rank.  Returns (loss [1]: the mean over all ranks' non-ignored rows, dX:
    this rank's rows, dW: summed over ranks unless reduce_dw is False,
    n_global [1] int64).  With dw_fp32 (the default) dW is fp32, written in
    fp32 by each rank and summed in fp32; otherwise it has X's dtype and the
    collective sums it in that dtype.  dw_slices = n > 0: dW reduced in n
    vocabulary slices, each as soon as it is final (overlapping the rest of
    the computation); dw_shard: reduce-scattered instead, one slice per rank,
    and the returned dW is this rank's rows [a, b) of the sum
    (binding.dw_slice_bounds(V, world)[rank]).
    """
    if reduce_dw and (dw_slices > 0 or dw_shard):
        n_sl = dist.get_world_size(group) if dw_shard else dw_slices
        bounds = binding.dw_slice_bounds(W.shape[0], n_sl)
        return data_parallel_step_sliced(
            lambda: binding.count_valid(X, W, labels, ignore_index, shift_seq_len=shift_seq_len),
            lambda n, ev: binding.fused(X, W, labels, ignore_index=ignore_index,
                                        softcap=softcap, dloss=dloss, ws=ws, n_valid_global=n,
                                        shift_seq_len=shift_seq_len, dw_fp32=dw_fp32,
                                        slice_events=ev),
            bounds, group=group, shard=dw_shard)
    return data_parallel_step(
        lambda: binding.count_valid(X, W, labels, ignore_index, shift_seq_len=shift_seq_len),
        lambda n: binding.fused(X, W, labels, ignore_index=ignore_index, softcap=softcap,
                                dloss=dloss, ws=ws, n_valid_global=n,
                                shift_seq_len=shift_seq_len, dw_fp32=dw_fp32),
        group=group, reduce_dw=reduce_dw)
