"""Row strides of X, W, dX and dW (flce_problem_t.ldx / ldw / lddx / lddw).

Callers pass views straight through instead of making the copies torchtune
issue #1228's recipe makes (``.contiguous()`` after slicing) and Liger-Kernel
issue #227 counts as fusable overhead: hidden states that are a column slice
of a wider activation, every other row of a buffer, a weight with padding
columns, gradients written into slices of wider buffers.  The kernels read
the same tiles whatever the row pitch, so a strided call equals the dense
call bit for bit; the columns past H of the output buffers are never
written; and the results match the oracle."""
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
from linear_cross_entropy_tiles_b200 import inputs
from parity import TOL, rel_fro, rel_scalar, run_oracle, to_np

pytestmark = pytest.mark.gpu

SCHEDULES = {"recompute": flce.FLCE_SCHEDULE_RECOMPUTE,
             "fused_fwd": flce.FLCE_SCHEDULE_FUSED_FORWARD}


class _schedule:
    def __init__(self, which):
        self.which = which

    def __enter__(self):
        self.prev = flce.flce_set_schedule(self.which)

    def __exit__(self, *exc):
        flce.flce_set_schedule(self.prev)


def _embed(t, pad, fill=float("nan"), every=1):
    """A view of t inside a larger buffer: `pad` extra columns per row and
    `every`-th rows (the rows between hold garbage)."""
    R, C = t.shape
    big = torch.full((R * every, C + pad), fill, dtype=t.dtype, device=t.device)
    view = big[::every, :C]
    view.copy_(t)
    return big, view


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("dtype,BT,H,V,cap", [("bf16", 600, 192, 3000, 0.0),
                                              ("bf16", 300, 1096, 1000, 30.0),
                                              ("bf16", 200, 64, 40000, 0.0),
                                              ("fp32", 130, 64, 900, 5.0)])
def test_strided_views_equal_dense_and_oracle(sched, dtype, BT, H, V, cap, cuda_device):
    if dtype == "fp32" and sched == "fused_fwd":
        pytest.skip("fp32 problems always use the recompute schedule")
    x_std, w_std = (1.0, 0.05) if dtype == "bf16" else (0.5, 0.1)
    X, W, lab = inputs.make_inputs(BT, H, V, dtype, x_std, w_std, 0.1, seed=31)
    Xd, Wd, labd = X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device)
    with _schedule(SCHEDULES[sched]):
        ref = flce.fused(Xd, Wd, labd, softcap=cap, dloss=0.5)
        _, Xs = _embed(Xd, 16, every=2)          # every other row of a wider buffer
        _, Ws = _embed(Wd, 8)                   # padding columns
        dXbig, dXs = _embed(torch.zeros_like(Xd), 24, fill=3.0)
        dWbig, dWs = _embed(torch.zeros_like(Wd), 8, fill=3.0, every=3)
        loss, dX, dW = flce.fused(Xs, Ws, labd, softcap=cap, dloss=0.5, dX=dXs, dW=dWs)
        torch.cuda.synchronize()
    assert dX.data_ptr() == dXs.data_ptr() and dW.data_ptr() == dWs.data_ptr()
    assert loss.item() == ref[0].item()
    assert torch.equal(dXs, ref[1]) and torch.equal(dWs, ref[2])
    assert bool((dXbig[:, H:] == 3.0).all())                  # pads untouched
    assert bool((dWbig[:, H:] == 3.0).all()) and bool((dWbig[1::3] == 3.0).all())
    o = run_oracle(X, W, lab, softcap=cap, dloss=0.5)
    tol = TOL[dtype]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"]
    assert rel_fro(to_np(dXs), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dWs), o["dW"]) <= tol["grad"]


def test_strided_forward_backward_pair(cuda_device):
    """flce_forward / flce_backward with strided X and W equal the dense pair."""
    BT, H, V = 260, 128, 2000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, seed=32)
    Xd, Wd, labd = X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device)
    loss_a, lse_a = flce.forward(Xd, Wd, labd)
    _, Xs = _embed(Xd, 64)
    _, Ws = _embed(Wd, 8, every=2)
    loss_b, lse_b = flce.forward(Xs, Ws, labd)
    assert loss_a.item() == loss_b.item() and torch.equal(lse_a, lse_b)
    dl = torch.tensor([1.0], device=cuda_device)
    dX_a, dW_a = flce.backward(Xd, Wd, labd, lse_a, dl)
    dX_b, dW_b = flce.backward(Xs, Ws, labd, lse_b, dl)
    torch.cuda.synchronize()
    assert torch.equal(dX_a, dX_b) and torch.equal(dW_a, dW_b)


def test_llama_shaped_slices_and_shift(cuda_device):
    """The Llama-3 head's H and V at a small BT: hidden states taken as the
    first 4096 of 4160 columns of a wider activation, the weight as rows of
    a vocabulary-padded embedding table, token ids shifted by the op (no
    slicing of hidden states or labels at all)."""
    B, T, H, V = 2, 300, 4096, 128256
    X, W, ids = inputs.make_inputs(B * T, H, V, "bf16", 1.0, 0.02, 0.0, seed=33,
                                   device=cuda_device)
    act = torch.randn(B * T, H + 64, device=cuda_device).to(torch.bfloat16)
    act[:, :H] = X
    table = torch.zeros(V + 128, H, dtype=torch.bfloat16, device=cuda_device)
    table[:V] = W
    ref = flce.fused(X, W, ids, shift_seq_len=T)
    out = flce.fused(act[:, :H], table[:V], ids, shift_seq_len=T)
    torch.cuda.synchronize()
    assert out[0].item() == ref[0].item()
    assert torch.equal(out[1], ref[1]) and torch.equal(out[2], ref[2])
