"""flce_fused_noalloc: the fused loss and gradients for callers that cannot
allocate device memory themselves (a plugin whose host program owns all of
the GPU's memory, or a caller from another language that can only pass the
tensors it was given).  It takes no workspace; its scratch space is a fixed
64 MiB array inside the library, shared by every call on a device.

The GPU test calls it several times in a row through the C ABI, on problems
of different shapes and both schedules (the fused-in-forward one keeps an
fp32 dW running sum and dX split slabs in the array, the in-op label shift a
copy of the labels), so every call runs on scratch a different call left
behind.  Each result must equal flce_fused with an ordinary workspace bit
for bit: the same kernels run in the same order on the same data.  The file
is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
from linear_cross_entropy_tiles_b200 import binding, inputs


def test_rejects_problems_beyond_the_scratch_size():
    # Checked on the host before any GPU work: the Llama-3 LM-head problem
    # needs far more scratch than the fixed array holds.
    w = inputs.WORKLOADS["llama3_8b"]
    p = flce.make_problem(w.BT, w.H, w.V)
    a = 1 << 20  # never dereferenced: the call returns before touching memory
    st = binding.lib().flce_fused_noalloc(ctypes.byref(p), a, a, a, 1.0, a, a, a, None)
    assert st == 4  # FLCE_ERR_WORKSPACE_TOO_SMALL
    assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) > 64 << 20


# BT, H, V, softcap, shift_seq_len, seed: recompute (BT < 512) and
# fused-in-forward (BT >= 512: two row chunks, fp32 dW sum, dX split slabs)
CALLS = [(300, 192, 1000, 0.0, 0, 41),
         (1024, 256, 4000, 0.0, 0, 43),
         (200, 128, 3000, 30.0, 0, 42),
         (1024, 128, 2000, 10.0, 256, 44),
         (600, 192, 1000, 0.0, 0, 45)]


@pytest.mark.gpu
def test_noalloc_equals_fused_bitwise_on_calls_in_a_row(cuda_device):
    for BT, H, V, cap, T, seed in CALLS:
        X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, seed=seed,
                                       device=cuda_device)
        p = flce.make_problem(BT, H, V, X.dtype, softcap=cap, shift_seq_len=T)
        assert 0 < flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) <= 64 << 20
        # Reference: the existing entry point with its own workspace.
        ref = flce.fused(X, W, lab, softcap=cap, dloss=0.75, shift_seq_len=T)
        # The allocation-free entry point, through the C ABI.
        loss = torch.empty(1, dtype=torch.float32, device=cuda_device)
        dX, dW = torch.empty_like(X), torch.empty_like(W)
        binding.flce_fused_noalloc(p, X, W, lab, 0.75, loss, dX, dW)
        torch.cuda.synchronize()
        assert loss.item() == ref[0].item(), (BT, H, V)
        assert torch.equal(dX, ref[1]) and torch.equal(dW, ref[2]), (BT, H, V)
