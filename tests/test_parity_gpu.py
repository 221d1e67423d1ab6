"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small problems span several 128-row, 256-column and 64-deep tiles with
ragged tails; the degenerate cases (one row, V = 1, every row ignored, an
empty batch) and device-detected errors are covered too."""
import numpy as np
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
import oracle
from linear_cross_entropy_tiles_b200 import inputs
from parity import TOL, rel_fro, rel_scalar, run_oracle, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # BT, H, V, dtype, softcap, ignore_frac, seed
    (300, 192, 1000, "bf16", 0.0, 0.10, 1),
    (256, 128, 512, "bf16", 0.0, 0.0, 2),
    (129, 64, 257, "bf16", 30.0, 0.05, 3),
    (77, 72, 3000, "bf16", 2.0, 0.20, 4),
    (520, 256, 40000, "bf16", 0.0, 0.05, 5),   # two vocabulary chunks
    (64, 64, 512, "bf16", 0.0, 0.10, 6),
    (1, 8, 1, "bf16", 0.0, 0.0, 7),
    (3, 16, 2, "bf16", 5.0, 0.0, 8),
    (64, 64, 512, "fp32", 0.0, 0.10, 9),
    (100, 40, 300, "fp32", 5.0, 0.10, 10),
    (70, 24, 20000, "fp32", 0.0, 0.05, 11),   # two fp32 chunks
    (200, 1096, 3000, "bf16", 0.0, 0.10, 12),  # H > 1024: four epilogue warps, ragged K
    (96, 1536, 777, "bf16", 10.0, 0.05, 13),
    # two row chunks of the fused-in-forward schedule, the last one ragged
    (1100, 64, 3000, "bf16", 0.0, 0.05, 14),
    (1300, 128, 1500, "bf16", 15.0, 0.10, 15),
]


class schedule:
    """Run a block with the process-wide flce_fused schedule forced."""

    def __init__(self, which):
        self.which = which

    def __enter__(self):
        self.prev = flce.flce_set_schedule(self.which)

    def __exit__(self, *exc):
        flce.flce_set_schedule(self.prev)


SCHEDULES = {"recompute": flce.FLCE_SCHEDULE_RECOMPUTE,
             "fused_fwd": flce.FLCE_SCHEDULE_FUSED_FORWARD}


def _inputs(BT, H, V, dtype, ignore_frac, seed, device):
    x_std, w_std = (1.0, 0.05) if dtype == "bf16" else (0.5, 0.1)
    X, W, lab = inputs.make_inputs(BT, H, V, dtype, x_std, w_std, ignore_frac, seed)
    return X, W, lab, X.to(device), W.to(device), lab.to(device)


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%dx%d-%s-cap%g" % c[:5])
def test_fused_matches_oracle(case, sched, cuda_device):
    BT, H, V, dtype, softcap, ign, seed = case
    if dtype == "fp32" and sched == "fused_fwd":
        pytest.skip("fp32 problems always use the recompute schedule")
    X, W, lab, Xd, Wd, labd = _inputs(BT, H, V, dtype, ign, seed, cuda_device)
    o = run_oracle(X, W, lab, softcap=softcap, dloss=0.5)
    with schedule(SCHEDULES[sched]):
        loss, dX, dW = flce.fused(Xd, Wd, labd, softcap=softcap, dloss=0.5)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"], (loss.item(), o["loss"])
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]


@pytest.mark.parametrize("case", CASES[:5] + CASES[8:10] + CASES[11:], ids=lambda c: "%dx%dx%d-%s-cap%g" % c[:5])
def test_forward_backward_match_oracle_and_fused(case, cuda_device):
    BT, H, V, dtype, softcap, ign, seed = case
    X, W, lab, Xd, Wd, labd = _inputs(BT, H, V, dtype, ign, seed, cuda_device)
    o = run_oracle(X, W, lab, softcap=softcap, dloss=1.0)
    p = flce.make_problem(BT, H, V, Xd.dtype, softcap=softcap)
    ws = flce.workspace(p, flce.FLCE_OP_FORWARD, cuda_device)
    loss, lse = flce.forward(Xd, Wd, labd, softcap=softcap, ws=ws)
    st, nv = flce.flce_get_device_status(ws)
    assert st == 0 and nv == o["n_valid"]          # labels / ignore mask: exact
    tol = TOL[dtype]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"]
    lse_err = np.max(np.abs(to_np(lse) - o["lse"]) / np.maximum(1.0, np.abs(o["lse"])))
    assert lse_err <= tol["lse"], lse_err
    dl = torch.tensor([1.0], device=cuda_device)
    dX, dW = flce.backward(Xd, Wd, labd, lse, dl, softcap=softcap)
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]
    # the recompute schedule of the fused call runs the same kernels in the
    # same order: bitwise equal
    with schedule(flce.FLCE_SCHEDULE_RECOMPUTE):
        l2, dX2, dW2 = flce.fused(Xd, Wd, labd, softcap=softcap, dloss=1.0)
    assert l2.item() == loss.item()
    assert torch.equal(dX2, dX) and torch.equal(dW2, dW)


@pytest.mark.parametrize("sched", list(SCHEDULES))
def test_deterministic_bitwise(sched, cuda_device):
    X, W, lab, Xd, Wd, labd = _inputs(333, 128, 5000, "bf16", 0.1, 21, cuda_device)
    with schedule(SCHEDULES[sched]):
        a = flce.fused(Xd, Wd, labd, softcap=10.0)
        b = flce.fused(Xd, Wd, labd, softcap=10.0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("sched", list(SCHEDULES))
def test_all_rows_ignored(sched, cuda_device):
    X, W, lab, Xd, Wd, labd = _inputs(200, 64, 700, "bf16", 0.0, 22, cuda_device)
    labd.fill_(-100)
    with schedule(SCHEDULES[sched]):
        loss, dX, dW = flce.fused(Xd, Wd, labd)
    assert loss.item() == 0.0
    assert torch.count_nonzero(dX).item() == 0 and torch.count_nonzero(dW).item() == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_empty_batch(dtype, cuda_device):
    dt = inputs.torch_dtype(dtype)
    Xd = torch.empty(0, 64, dtype=dt, device=cuda_device)
    Wd = torch.randn(300, 64, device=cuda_device).to(dt)
    labd = torch.empty(0, dtype=torch.int64, device=cuda_device)
    loss, dX, dW = flce.fused(Xd, Wd, labd)
    assert loss.item() == 0.0 and dX.shape == (0, 64)
    assert torch.count_nonzero(dW).item() == 0


def test_ignore_index_value(cuda_device):
    X, W, lab, Xd, Wd, labd = _inputs(150, 64, 900, "bf16", 0.0, 23, cuda_device)
    lab[::3] = 7
    labd = lab.to(cuda_device)
    o = run_oracle(X, W, lab, ignore_index=7)
    loss, dX, dW = flce.fused(Xd, Wd, labd, ignore_index=7)
    assert rel_scalar(loss.item(), o["loss"]) <= 2e-3
    assert rel_fro(to_np(dX), o["dX"]) <= 1e-2 and rel_fro(to_np(dW), o["dW"]) <= 1e-2


@pytest.mark.parametrize("bad", [900, -1, 10 ** 12])
def test_bad_label_reported_on_device(bad, cuda_device):
    X, W, lab, Xd, Wd, labd = _inputs(130, 64, 900, "bf16", 0.0, 24, cuda_device)
    labd[77] = bad
    p = flce.make_problem(130, 64, 900)
    ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
    loss = torch.empty(1, device=cuda_device)
    dX, dW = torch.empty_like(Xd), torch.empty_like(Wd)
    flce.flce_fused(p, Xd, Wd, labd, 1.0, loss, dX, dW, ws)
    st, _ = flce.flce_get_device_status(ws)
    assert st == 5
    # the next call on the same workspace starts clean
    labd[77] = 3
    flce.flce_fused(p, Xd, Wd, labd, 1.0, loss, dX, dW, ws)
    assert flce.flce_get_device_status(ws)[0] == 0


def test_launch_count_and_stream(cuda_device):
    X, W, lab, Xd, Wd, labd = _inputs(256, 128, 2000, "bf16", 0.0, 25, cuda_device)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        loss, dX, dW = flce.fused(Xd, Wd, labd, stream=s)
    n = flce.flce_last_launch_count()
    assert n == 1 + 3 + 3  # labels, LSE GEMM, combine, finalize, one chunk of 3 GEMMs
    s.synchronize()
    ref = flce.fused(Xd, Wd, labd)
    assert torch.equal(ref[1], dX)
    with schedule(flce.FLCE_SCHEDULE_FUSED_FORWARD):
        flce.flce_profile_start(64)
        flce.fused(Xd, Wd, labd)
        n = flce.flce_last_launch_count()
        names = [k for k, _ in flce.flce_profile_stop()]
    # labels, 2 row chunks x (forward GEMM, lse_q, recomputation GEMM (returns
    # at once: nothing flagged), lse_q, dX GEMM [+ split reduce], dW GEMM),
    # finalize
    assert len(names) == n
    chunk = ["lse_q_gemm", "lse_q", "lse_q_repair_gemm", "lse_q", "dx_gemm"]
    tail = ["dw_acc_gemm"]
    body = names[1:-1]
    if "dx_reduce" in body:
        tail = ["dx_reduce"] + tail
    assert names[0] == "labels" and names[-1] == "loss_finalize"
    assert body == (chunk + tail) * 2


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    """A wait that nothing satisfies gives up after its limit (here 50 ms),
    records FLCE_ERR_TIMEOUT, and the next call on the same workspace runs
    normally and clears it."""
    X, W, lab, Xd, Wd, labd = _inputs(130, 64, 900, "bf16", 0.0, 26, cuda_device)
    p = flce.make_problem(130, 64, 900)
    ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
    flce.flce_selftest_wait_timeout(ws, 50_000_000)
    assert flce.flce_get_device_status(ws)[0] == 6
    loss = torch.empty(1, device=cuda_device)
    dX, dW = torch.empty_like(Xd), torch.empty_like(Wd)
    flce.flce_fused(p, Xd, Wd, labd, 1.0, loss, dX, dW, ws)
    assert flce.flce_get_device_status(ws)[0] == 0
    assert torch.equal(flce.fused(Xd, Wd, labd)[1], dX)


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("V", [128, 129, 255, 256, 257, 383, 384, 385, 50257])
def test_vocab_edges(V, sched, cuda_device):
    """Vocabulary sizes around the 128- and 256-column tile edges, where the
    last tile's upper half may hold no vocabulary column at all."""
    X, W, lab, Xd, Wd, labd = _inputs(300, 64, V, "bf16", 0.1, 27, cuda_device)
    o = run_oracle(X, W, lab, dloss=1.0)
    with schedule(SCHEDULES[sched]):
        loss, dX, dW = flce.fused(Xd, Wd, labd)
    torch.cuda.synchronize()
    assert rel_scalar(loss.item(), o["loss"]) <= 2e-3
    assert rel_fro(to_np(dX), o["dX"]) <= 1e-2 and rel_fro(to_np(dW), o["dW"]) <= 1e-2


@pytest.mark.parametrize("H", [64, 1096])
def test_wide_logit_spread_within_a_tile(H, cuda_device):
    """The forward epilogue takes its exponent reference from the first 32
    columns of each 128- or 256-column range; here those columns sit about
    100 nats below the rest, so the one-pass sums overflow and the exact
    two-pass path must redo the range.  Results still match the oracle."""
    BT, V = 600, 1000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.05, 41)
    X[:, 0] = 1.0
    W[:, 0] = 0.0
    first = (torch.arange(V) % 128) < 32
    W[first, 0] = -100.0
    o = run_oracle(X, W, lab, dloss=1.0)
    with schedule(SCHEDULES["fused_fwd"]):
        loss, dX, dW = flce.fused(X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device))
    torch.cuda.synchronize()
    assert np.isfinite(to_np(dX)).all() and np.isfinite(to_np(dW)).all()
    assert rel_scalar(loss.item(), o["loss"]) <= TOL["bf16"]["loss"]
    assert rel_fro(to_np(dX), o["dX"]) <= TOL["bf16"]["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= TOL["bf16"]["grad"]


@pytest.mark.parametrize("sched", list(SCHEDULES))
@pytest.mark.parametrize("B,T,cap", [(3, 101, 0.0), (2, 256, 30.0), (5, 1, 0.0)])
def test_in_op_label_shift(B, T, cap, sched, cuda_device):
    """shift_seq_len = T: labels are the token ids of B sequences and the op
    scores position t against id t+1 itself (the last position of each
    sequence is ignored), so callers pass hidden states and ids without
    slicing or copying.  Matches the oracle given the shifted labels; the
    forward/backward pair agrees too; N_valid is exact."""
    BT, H, V = B * T, 64, 1000
    X, W, ids = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, 71)
    lab = torch.cat([ids.reshape(B, T)[:, 1:],
                     torch.full((B, 1), inputs.IGNORE_INDEX, dtype=ids.dtype)], 1).reshape(-1)
    if int((lab != inputs.IGNORE_INDEX).sum()) == 0:
        o = None
    else:
        o = run_oracle(X, W, lab, softcap=cap, dloss=0.5)
    Xd, Wd, idsd = X.to(cuda_device), W.to(cuda_device), ids.to(cuda_device)
    with schedule(SCHEDULES[sched]):
        p = flce.make_problem(BT, H, V, Xd.dtype, softcap=cap, shift_seq_len=T)
        ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
        loss, dX, dW = flce.fused(Xd, Wd, idsd, softcap=cap, dloss=0.5, ws=ws, shift_seq_len=T)
        status, nv = flce.flce_get_device_status(ws)
    assert status == 0 and nv == oracle.count_valid(lab.numpy())
    if o is None:  # T = 1: every position is the last of its sequence
        assert loss.item() == 0.0 and not dX.any() and not dW.any()
        return
    tol = TOL["bf16"]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"]
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]
    loss_f, lse = flce.forward(Xd, Wd, idsd, softcap=cap, shift_seq_len=T)
    dl = torch.full((1,), 0.5, device=cuda_device)
    dX2, dW2 = flce.backward(Xd, Wd, idsd, lse, dl, softcap=cap, shift_seq_len=T)
    assert rel_scalar(loss_f.item(), o["loss"]) <= tol["loss"]
    assert rel_fro(to_np(dX2), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW2), o["dW"]) <= tol["grad"]


@pytest.mark.parametrize("sched", list(SCHEDULES))
def test_cuda_graph_capture_and_replay(sched, cuda_device):
    """flce_fused allocates nothing and never waits on the host, so a whole
    call can be captured into a CUDA graph; replays give the eager results
    bit for bit, also after the inputs change in place."""
    BT, H, V = 600, 128, 3000
    X, W, lab, Xd, Wd, labd = _inputs(BT, H, V, "bf16", 0.05, 81, cuda_device)
    with schedule(SCHEDULES[sched]):
        p = flce.make_problem(BT, H, V, Xd.dtype)
        ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
        loss = torch.empty(1, dtype=torch.float32, device=cuda_device)
        dX, dW = torch.empty_like(Xd), torch.empty_like(Wd)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # warm-up off the capture (first-use setup)
            flce.flce_fused(p, Xd, Wd, labd, 1.0, loss, dX, dW, ws, side)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            flce.flce_fused(p, Xd, Wd, labd, 1.0, loss, dX, dW, ws)
        for _ in range(2):
            g.replay()
            torch.cuda.synchronize()
            ref = flce.fused(Xd, Wd, labd)
            assert torch.equal(loss, ref[0]) and torch.equal(dX, ref[1])
            assert torch.equal(dW, ref[2])
            Xd.mul_(0.5)  # new inputs in the same buffers


@pytest.mark.parametrize("cap", [0.0, 60.0])
@pytest.mark.parametrize("H", [64, 1096])
def test_rows_outside_the_shared_reference_range(cap, H, cuda_device):
    """The fused-in-forward schedule stores q = exp(y - R) against one
    reference R = 0 per row.  Rows whose logits all sit near +80 nats (one
    near +200, where the sums overflow) or near -80 nats leave the range that
    keeps q and the prescaled X in bf16; they are flagged, their 32-row
    groups recomputed against each row's own maximum, and the other rows of
    those groups and tiles finished again with the same values.  Ignored
    rows are never flagged.  Everything matches the oracle."""
    BT, V = 700, 3000
    X, W, lab = inputs.make_inputs(BT, H, V, "bf16", 1.0, 0.05, 0.1, 91)
    W[:, 0] = 1.0     # X[i, 0] now shifts every logit of row i
    X[:, 0] = 0.0
    high, low = [5, 300, 301, 650], [70, 71, 400, 699]
    X[high, 0] = 80.0
    X[low, 0] = -80.0
    X[130, 0] = 200.0
    lab[[5, 71]] = inputs.IGNORE_INDEX
    o = run_oracle(X, W, lab, softcap=cap, dloss=0.5)
    with schedule(SCHEDULES["fused_fwd"]):
        loss, dX, dW = flce.fused(X.to(cuda_device), W.to(cuda_device), lab.to(cuda_device),
                                  softcap=cap, dloss=0.5)
    torch.cuda.synchronize()
    assert torch.isfinite(dX).all() and torch.isfinite(dW).all()
    tol = TOL["bf16"]
    assert rel_scalar(loss.item(), o["loss"]) <= tol["loss"], (loss.item(), o["loss"])
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]
    # row by row: the recomputed rows and their group neighbours
    for i in high + low + [130, 131, 301, 64]:
        ref = o["dX"][i]
        nrm = np.linalg.norm(ref)
        got = to_np(dX[i:i + 1])[0]
        assert (nrm == 0 and not got.any()) or np.linalg.norm(got - ref) <= 2e-2 * nrm, i
