"""dW in fp32 (flce_problem_t.dw_fp32 = 1) for bf16 inputs, and the
workspace cap of the automatic schedule.

An fp32 dW is what a data-parallel job sums over ranks (each rank's G^T X
kept at fp32 until the cross-rank sum) and what mixed-precision optimisers
keep; in the fused-in-forward schedule it also holds the running sum over
row chunks, so the workspace loses its V x H fp32 array.  Both schedules
compute the same fp32 sums as with a bf16 dW and only skip the final
rounding: rounded to bf16, the fp32 dW equals the bf16 dW bit for bit."""
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


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("BT,H,V,cap", [(600, 192, 3000, 0.0), (300, 1096, 1000, 30.0),
                                        (200, 64, 40000, 0.0), (1300, 256, 777, 5.0)])
def test_fp32_dW_rounds_to_the_bf16_dW(sched, BT, H, V, cap, cuda_device):
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, seed=51, device=cuda_device)
    with _schedule(SCHEDULES[sched]):
        l16, dX16, dW16 = flce.fused(X, W, lab, softcap=cap, dloss=0.5)
        l32, dX32, dW32 = flce.fused(X, W, lab, softcap=cap, dloss=0.5, dw_fp32=True)
        # an fp32 dW inside a wider buffer (row stride H + 4 floats)
        big = torch.full((V, H + 4), 3.0, dtype=torch.float32, device=cuda_device)
        l3, dX3, dW3 = flce.fused(X, W, lab, softcap=cap, dloss=0.5, dW=big[:, :H])
        torch.cuda.synchronize()
    assert dW32.dtype == torch.float32
    assert l32.item() == l16.item() and torch.equal(dX32, dX16)
    assert torch.equal(dW32.to(torch.bfloat16), dW16)
    assert torch.equal(dW3, dW32) and bool((big[:, H:] == 3.0).all())
    o = run_oracle(X.cpu(), W.cpu(), lab.cpu(), softcap=cap, dloss=0.5)
    assert rel_scalar(l32.item(), o["loss"]) <= TOL["bf16"]["loss"]
    assert rel_fro(to_np(dW32), o["dW"]) <= TOL["bf16"]["grad"]


def test_fp32_dW_forward_backward_pair(cuda_device):
    BT, H, V = 300, 128, 5000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, seed=52, device=cuda_device)
    loss, lse = flce.forward(X, W, lab)
    dl = torch.tensor([1.0], device=cuda_device)
    dX16, dW16 = flce.backward(X, W, lab, lse, dl)
    p = flce.make_problem(BT, H, V, X.dtype, dw_fp32=1)
    ws = flce.workspace(p, flce.FLCE_OP_BACKWARD, cuda_device)
    dX32 = torch.empty_like(X)
    dW32 = torch.empty(V, H, dtype=torch.float32, device=cuda_device)
    flce.flce_backward(p, X, W, lab, lse, dl, dX32, dW32, ws)
    torch.cuda.synchronize()
    assert torch.equal(dX32, dX16) and torch.equal(dW32.to(torch.bfloat16), dW16)


@pytest.mark.parametrize("cap_kind", ["logits", "tiny"])
def test_workspace_cap_keeps_results(cap_kind, cuda_device):
    """Under a cap the automatic schedule switches to the recompute plan (and
    narrows its vocabulary chunk for the tiny cap): results match the oracle,
    and the workspace the caller allocates is the capped size."""
    # H > BT / 2: the fused-in-forward plan's fp32 dW sum (V x H) alone is
    # larger than one bf16 BT x V tensor, so the logits-sized cap rejects it
    BT, H, V = 1024, 1024, 6000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, seed=53, device=cuda_device)
    p = flce.make_problem(BT, H, V, X.dtype)
    cap = 2 * BT * V if cap_kind == "logits" else 1
    prev = flce.flce_set_workspace_limit(cap)
    try:
        n = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
        loss, dX, dW = flce.fused(X, W, lab)
        torch.cuda.synchronize()
    finally:
        flce.flce_set_workspace_limit(prev)
    free = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
    assert n < free and (cap_kind == "tiny" or n <= cap)
    o = run_oracle(X.cpu(), W.cpu(), lab.cpu())
    assert rel_scalar(loss.item(), o["loss"]) <= TOL["bf16"]["loss"]
    assert rel_fro(to_np(dX), o["dX"]) <= TOL["bf16"]["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= TOL["bf16"]["grad"]
