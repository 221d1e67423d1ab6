"""Vocabulary-parallel FLCE: one process per GPU, each holding a slice of
the vocabulary (rows [v_offset, v_offset + V_r) of W) and all of X and the
labels.

The mean loss needs each row's log-sum-exp over the whole vocabulary, so a
step exchanges:

  1. after the forward, every rank's per-row (max, sum-exp, label logit)
     over its slice (flce_vp_forward): an all-gather of 3 floats per row;
     every rank then combines them in rank order into the same lse and loss
     (flce_vp_combine);
  2. after the backward (flce_vp_backward, from the global lse): the sum over
     ranks of their fp32 shares of dX (an all-reduce of BT x H floats).
     dW stays with its rank: its rows of the vocabulary.

All arithmetic runs in the library's kernels; torch.distributed (NCCL on
GPUs) carries the exchanges.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding


def vp_offsets(v_total: int, world: int):
    """Contiguous vocabulary slices, as even as possible: [(offset, rows)]."""
    base, extra = divmod(int(v_total), int(world))
    out, off = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((off, n))
        off += n
    return out


def vocab_parallel_step(forward_stats, combine, backward, group=None):
    """The exchange pattern of a vocabulary-parallel FLCE step.

    forward_stats() returns this rank's stats [BT, 3]; combine(stats_all
    [world, BT, 3]) returns (loss [1], lse [BT]); backward(lse) returns (this
    rank's dX share [BT, H], its dW rows).  Returns (loss, lse, dX summed
    over the ranks, dW rows).  Every rank must call it the same number of
    times, in the same order.
    """
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    stats = forward_stats()
    if world > 1:
        flat = torch.empty((world * stats.shape[0],) + tuple(stats.shape[1:]),
                           dtype=stats.dtype, device=stats.device)
        dist.all_gather_into_tensor(flat, stats.contiguous(), group=group)
        stats_all = flat.view((world,) + tuple(stats.shape))
    else:
        stats_all = stats.reshape((1,) + tuple(stats.shape))
    loss, lse = combine(stats_all)
    dX, dW = backward(lse)
    if world > 1:
        dist.all_reduce(dX, op=dist.ReduceOp.SUM, group=group)
    return loss, lse, dX, dW


def fused_vp(X: torch.Tensor, W_r: torch.Tensor, labels: torch.Tensor, v_offset: int,
             v_total: int, group=None, ignore_index: int = -100, softcap: float = 0.0,
             dloss: float = 1.0):
    """Forward and backward of FLCE with W split over the vocabulary.

    X [BT, H] and labels [BT] (global ids) are the same on every rank; W_r
    [V_r, H] is this rank's slice starting at vocabulary id v_offset.
    Returns (loss [1], lse [BT], dX fp32 [BT, H] summed over the ranks, dW_r:
    the gradient of this rank's rows of W).  Every rank must call it with
    the same X, labels and v_total, in the same order.
    """
    dev = X.device
    BT, H = X.shape
    p = binding._problem_of(X, W_r, ignore_index, softcap)
    ws_f = torch.empty(binding.flce_vp_workspace_size(p, binding.FLCE_OP_FORWARD),
                       dtype=torch.uint8, device=dev)

    def forward_stats():
        stats = torch.empty(BT, 3, dtype=torch.float32, device=dev)
        binding.flce_vp_forward(p, v_offset, v_total, X, W_r, labels, stats, ws_f)
        return stats

    def combine(stats_all):
        pg = binding.make_problem(BT, H, v_total, X.dtype, ignore_index, softcap)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        lse = torch.empty(BT, dtype=torch.float32, device=dev)
        binding.flce_vp_combine(pg, stats_all.shape[0], stats_all, labels, loss, lse, ws_f)
        return loss, lse

    def backward(lse):
        ws_b = torch.empty(binding.flce_vp_workspace_size(p, binding.FLCE_OP_BACKWARD),
                           dtype=torch.uint8, device=dev)
        dX = torch.empty(BT, H, dtype=torch.float32, device=dev)
        dW = torch.empty_like(W_r)
        dl = torch.full((1,), float(dloss), dtype=torch.float32, device=dev)
        binding.flce_vp_backward(p, v_offset, v_total, X, W_r, labels, lse, dl, dX, dW, ws_b)
        return dX, dW

    return vocab_parallel_step(forward_stats, combine, backward, group=group)
