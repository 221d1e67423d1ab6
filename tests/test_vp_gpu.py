"""Vocabulary parallelism on one GPU: R ranks emulated in one process, each
running flce_vp_forward / flce_vp_backward on its slice of W, their
statistics stacked in rank order for flce_vp_combine, their fp32 dX shares
summed; the result against the oracle on the whole vocabulary.  Slices are
uneven and not multiples of the 256-column tile; labels fall in every slice;
ignored rows and the softcap are covered.  Then vp.fused_vp over a one-rank
NCCL group."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
from linear_cross_entropy_tiles_b200 import binding, inputs, vp
from parity import TOL, rel_fro, rel_scalar, run_oracle, to_np

pytestmark = pytest.mark.gpu


def _emulate(X, W, lab, slices, cap, dloss, dev):
    BT, H = X.shape
    V = W.shape[0]
    stats, shares = [], []
    for off, n in slices:
        W_r = W[off:off + n]
        p = binding._problem_of(X, W_r, -100, cap)
        ws = torch.empty(flce.binding.flce_vp_workspace_size(p, flce.FLCE_OP_FORWARD),
                         dtype=torch.uint8, device=dev)
        st = torch.empty(BT, 3, dtype=torch.float32, device=dev)
        binding.flce_vp_forward(p, off, V, X, W_r, lab, st, ws)
        stats.append(st)
    stats_all = torch.stack(stats).contiguous()
    pg = flce.make_problem(BT, H, V, X.dtype, softcap=cap)
    ws = torch.empty(256 + 2 * ((4 * BT + 255) // 256) * 256, dtype=torch.uint8, device=dev)
    loss = torch.empty(1, device=dev)
    lse = torch.empty(BT, device=dev)
    binding.flce_vp_combine(pg, len(slices), stats_all, lab, loss, lse, ws)
    dl = torch.tensor([dloss], device=dev)
    dX = torch.zeros(BT, H, dtype=torch.float64, device=dev)
    dWs = []
    for off, n in slices:
        W_r = W[off:off + n]
        p = binding._problem_of(X, W_r, -100, cap)
        ws = torch.empty(flce.binding.flce_vp_workspace_size(p, flce.FLCE_OP_BACKWARD),
                         dtype=torch.uint8, device=dev)
        dx = torch.empty(BT, H, dtype=torch.float32, device=dev)
        dw = torch.empty_like(W_r)
        binding.flce_vp_backward(p, off, V, X, W_r, lab, lse, dl, dx, dw, ws)
        dX += dx.double()          # the all-reduce of the shares (test-side)
        dWs.append(dw)
    torch.cuda.synchronize()
    return loss, lse, dX, torch.cat(dWs)


@pytest.mark.parametrize("dtype,cap,R", [("bf16", 0.0, 3), ("bf16", 30.0, 4), ("fp32", 5.0, 3),
                                         ("bf16", 0.0, 1)])
def test_vocab_parallel_emulated_matches_oracle(dtype, cap, R, cuda_device):
    BT, H, V = 300, 192, 3001
    x_std, w_std = (1.0, 0.05) if dtype == "bf16" else (0.5, 0.1)
    X, W, lab = inputs.make_inputs(BT, H, V, dtype, x_std, w_std, 0.1, seed=77)
    slices = vp.vp_offsets(V, R)
    Xd, Wd, labd = X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device)
    loss, lse, dX, dW = _emulate(Xd, Wd, labd, slices, cap, 0.5, cuda_device)
    o = run_oracle(X, W, lab, softcap=cap, dloss=0.5)
    tol = TOL[dtype]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"]
    lse_err = np.max(np.abs(to_np(lse) - o["lse"]) / np.maximum(1.0, np.abs(o["lse"])))
    assert lse_err <= tol["lse"], lse_err
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]
    # the unsplit forward's lse agrees to fp32 rounding
    _, lse1 = flce.forward(Xd, Wd, labd, softcap=cap)
    assert float(((lse - lse1).abs() / lse1.abs().clamp_min(1.0)).max()) <= 1e-6


def test_vocab_parallel_labels_checked_against_the_whole_vocabulary(cuda_device):
    BT, H, V = 64, 64, 1000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.0, seed=78, device=cuda_device)
    W_r = W[500:]
    p = binding._problem_of(X, W_r, -100, 0.0)
    ws = torch.empty(flce.binding.flce_vp_workspace_size(p, flce.FLCE_OP_FORWARD),
                     dtype=torch.uint8, device=cuda_device)
    st = torch.empty(BT, 3, device=cuda_device)
    binding.flce_vp_forward(p, 500, V, X, W_r, lab, st, ws)   # labels in [0, 1000): fine
    assert flce.flce_get_device_status(ws)[0] == 0
    lab[5] = V
    binding.flce_vp_forward(p, 500, V, X, W_r, lab, st, ws)
    assert flce.flce_get_device_status(ws)[0] == 5


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_fused_vp_one_rank_nccl(cuda_device):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=cuda_device)
    try:
        X, W, lab = inputs.make_inputs(700, 128, 2500, "bf16", 1.0, 0.05, 0.05, 79,
                                       device=cuda_device)
        loss, lse, dX, dW = vp.fused_vp(X, W, lab, 0, 2500, softcap=10.0)
        l1, lse1, dX1, dW1 = _emulate(X, W, lab, [(0, 2500)], 10.0, 1.0, cuda_device)
        torch.cuda.synchronize()
        assert torch.equal(loss, l1) and torch.equal(lse, lse1)
        assert torch.equal(dX.double(), dX1) and torch.equal(dW, dW1)
    finally:
        dist.destroy_process_group()
