"""The data-parallel entry points on one GPU: flce_count_valid against the
oracle's count (exact), flce_fused_global against the oracle with the same
global divisor, and dp.fused_dp over a one-rank NCCL group against
flce_fused (bit for bit: the collectives of one rank are identities)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
import oracle
from linear_cross_entropy_tiles_b200 import dp, inputs
from parity import TOL, rel_fro, rel_scalar, run_oracle, to_np

pytestmark = pytest.mark.gpu


def _shift(ids, T, ignore=-100):
    """Host-side shift (test reference): row (b, t) -> id (b, t+1), last position ignored."""
    x = ids.reshape(-1, T)
    return torch.cat([x[:, 1:], torch.full_like(x[:, :1], ignore)], dim=1).reshape(-1)


@pytest.mark.parametrize("BT,ign,T", [(0, 0.0, 0), (1, 0.0, 0), (300, 0.1, 0), (5000, 0.05, 0),
                                      (777, 1.0, 0), (300, 0.1, 100), (5000, 0.05, 1),
                                      (4096, 0.0, 1024)])
def test_count_valid_exact(BT, ign, T, cuda_device):
    _, _, lab = inputs.make_inputs(max(BT, 1), 8, 100, "bf16", 1.0, 0.05, ign, 61)
    lab = lab[:BT]
    X = torch.empty(BT, 8, dtype=torch.bfloat16, device=cuda_device)
    W = torch.empty(100, 8, dtype=torch.bfloat16, device=cuda_device)
    n = flce.count_valid(X, W, lab.to(cuda_device), shift_seq_len=T)
    ref = _shift(lab, T) if T else lab
    assert int(n.item()) == oracle.count_valid(ref.numpy())


@pytest.mark.parametrize("sched", ["recompute", "fused_fwd"])
@pytest.mark.parametrize("extra", [0, 37])
def test_fused_global_matches_oracle(sched, extra, cuda_device):
    """A rank's share: its rows' NLL summed over N_global = its own count
    plus `extra` rows held by other ranks; dX, dW scaled the same way."""
    BT, H, V, cap = 600, 192, 3000, 10.0
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, 62)
    n_global = oracle.count_valid(lab.numpy()) + extra
    o = run_oracle(X, W, lab, softcap=cap, n_valid=n_global, dloss=0.5)
    nd = torch.tensor([n_global], dtype=torch.int64, device=cuda_device)
    prev = flce.flce_set_schedule({"recompute": flce.FLCE_SCHEDULE_RECOMPUTE,
                                   "fused_fwd": flce.FLCE_SCHEDULE_FUSED_FORWARD}[sched])
    try:
        p = flce.make_problem(BT, H, V, torch.bfloat16, softcap=cap)
        ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
        loss, dX, dW = flce.fused(X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device),
                                  softcap=cap, dloss=0.5, ws=ws, n_valid_global=nd)
        status, nv = flce.flce_get_device_status(ws)
    finally:
        flce.flce_set_schedule(prev)
    assert status == 0 and nv == n_global
    tol = TOL["bf16"]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"]
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]


def test_fused_global_zero_count(cuda_device):
    X, W, lab = inputs.make_inputs(300, 64, 500, "bf16", 1.0, 0.05, 0.0, 63)
    nd = torch.zeros(1, dtype=torch.int64, device=cuda_device)
    loss, dX, dW = flce.fused(X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device),
                              n_valid_global=nd)
    assert loss.item() == 0.0
    assert not dX.any() and not dW.any()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_fused_dp_one_rank_nccl_equals_fused(cuda_device):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    try:
        X, W, lab = inputs.make_inputs(900, 128, 2000, "bf16", 1.0, 0.05, 0.05, 64,
                                       device=cuda_device)
        loss, dX, dW, n = dp.fused_dp(X, W, lab)
        ref = flce.fused(X, W, lab)
        torch.cuda.synchronize()
        assert int(n.item()) == int((lab != -100).sum().item())
        assert dW.dtype == torch.float32           # summed over ranks in fp32
        assert torch.equal(loss, ref[0]) and torch.equal(dX, ref[1])
        assert torch.equal(dW.to(torch.bfloat16), ref[2])
        l16, dX16, dW16, _ = dp.fused_dp(X, W, lab, dw_fp32=False)
        assert dW16.dtype == torch.bfloat16 and torch.equal(dW16, ref[2])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sched", ["recompute", "fused_fwd"])
@pytest.mark.parametrize("n_slices,dw_fp32", [(1, False), (4, False), (8, False), (3, True)])
def test_sliced_dW_equals_unsliced(sched, n_slices, dw_fp32, cuda_device):
    """flce_fused_global_sliced: the last row chunk's dW GEMM in vocabulary
    slices of whole 256-row tiles computes the same tiles in the same order,
    so loss, dX and dW equal flce_fused's bit for bit (V = 3000 in 8 slices
    of 512 rows leaves two empty); every slice's event is recorded; the
    fused-in-forward schedule launches one dW GEMM per non-empty slice in
    its last row chunk, and dW may be a row-strided view."""
    BT, H, V, cap = 1100, 128, 3000, 5.0
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, 65, device=cuda_device)
    prev = flce.flce_set_schedule({"recompute": flce.FLCE_SCHEDULE_RECOMPUTE,
                                   "fused_fwd": flce.FLCE_SCHEDULE_FUSED_FORWARD}[sched])
    try:
        ref = flce.fused(X, W, lab, softcap=cap, dloss=0.5, dw_fp32=dw_fp32)
        events = [torch.cuda.Event() for _ in range(n_slices)]
        dt = torch.float32 if dw_fp32 else torch.bfloat16
        big = torch.full((V, H + 8), 3.0, dtype=dt, device=cuda_device)
        flce.flce_profile_start(256)
        out = flce.fused(X, W, lab, softcap=cap, dloss=0.5, dW=big[:, :H], slice_events=events)
        names = [k for k, _ in flce.flce_profile_stop()]
    finally:
        flce.flce_set_schedule(prev)
    torch.cuda.synchronize()
    assert all(e.query() for e in events)
    assert torch.equal(out[0], ref[0]) and torch.equal(out[1], ref[1])
    assert torch.equal(out[2], ref[2]) and bool((big[:, H:] == 3.0).all())
    bounds = flce.dw_slice_bounds(V, n_slices)
    assert bounds[0][0] == 0 and bounds[-1][1] == V
    assert all(b0 == a1 for (_, b0), (a1, _) in zip(bounds, bounds[1:]))
    if sched == "fused_fwd":
        nonempty = sum(b > a for a, b in bounds)
        assert names.count("dw_acc_gemm") == names.count("lse_q_gemm") - 1 + nonempty


def test_fused_dp_sliced_and_sharded_one_rank_nccl(cuda_device):
    """dp.fused_dp reducing dW slice by slice on a side stream (all-reduce),
    or onto one rank per slice (reduce-scatter), over a one-rank NCCL group:
    equal to flce_fused bit for bit; the shard of the only rank is all of dW."""
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    try:
        X, W, lab = inputs.make_inputs(1100, 128, 3000, "bf16", 1.0, 0.05, 0.05, 66,
                                       device=cuda_device)
        ref = flce.fused(X, W, lab, dw_fp32=True)
        loss, dX, dW, n = dp.fused_dp(X, W, lab, dw_slices=3)
        l2, dX2, dW2, _ = dp.fused_dp(X, W, lab, dw_shard=True)
        torch.cuda.synchronize()
        assert int(n.item()) == int((lab != -100).sum().item())
        for lo, dx, dw in ((loss, dX, dW), (l2, dX2, dW2)):
            assert torch.equal(lo, ref[0]) and torch.equal(dx, ref[1])
            assert dw.shape == ref[2].shape and torch.equal(dw, ref[2])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("capped", [False, True])
def test_sliced_dW_with_shift_softcap_and_workspace_cap(capped, cuda_device):
    """The sliced hand-over composes with the in-op label shift and the
    softcap, and with a workspace cap that sends the automatic schedule to
    the recompute plan (whose events are all recorded after its last
    launch): equal to the unsliced call bit for bit in each case."""
    B, T, H, V, cap = 5, 240, 128, 3000, 20.0
    X, W, ids = inputs.make_inputs(B * T, H, V, "bf16", 1.0, 0.05, 0.0, 67, device=cuda_device)
    p = flce.make_problem(B * T, H, V, torch.bfloat16, softcap=cap, shift_seq_len=T)
    prev = flce.flce_set_workspace_limit(1 << 20 if capped else 0)
    try:
        ref = flce.fused(X, W, ids, softcap=cap, shift_seq_len=T)
        events = [torch.cuda.Event() for _ in range(5)]
        out = flce.fused(X, W, ids, softcap=cap, shift_seq_len=T, slice_events=events)
        ws_size = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
    finally:
        flce.flce_set_workspace_limit(prev)
    torch.cuda.synchronize()
    assert all(e.query() for e in events)
    for a, b in zip(out, ref):
        assert torch.equal(a, b)
    if capped:
        assert ws_size < 64 << 20  # the capped plan is the recompute schedule
