"""Parity at the workloads' full sizes, in the launch configuration bench.py
times (flce_fused, automatic schedule, CTA-pair kernels).

The oracle cannot redo a whole 8192 x 128256 x 4096 problem in seconds, so:
  * sampled rows: the full-size run's dX rows and forward lse rows are
    compared with the oracle on those rows (given the global N_valid);
  * N_valid (labels and ignore mask) is compared exactly;
  * the fused loss is compared with the separate forward kernel's loss;
  * without a softcap, every column of dW sums to zero over the vocabulary
    (softmax rows sum to one), a property of the full result;
  * determinism: a second call gives bit-identical results;
  * a row-subset problem (the sampled rows, the full W) is run through the
    GPU under both schedules and compared with the oracle on loss, dX and the
    whole dW.
"""
import numpy as np
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
import oracle
from linear_cross_entropy_tiles_b200 import inputs
from parity import TOL, rel_fro, rel_scalar, run_oracle, to_np

pytestmark = pytest.mark.gpu

FULL = ["gpt2_small", "llama3_8b", "gemma2_softcap"]
N_ROWS = 16


class _Schedule:
    def __init__(self, which):
        self.which = which

    def __enter__(self):
        self.prev = flce.flce_set_schedule(self.which)

    def __exit__(self, *exc):
        flce.flce_set_schedule(self.prev)


@pytest.fixture(scope="module")
def full_runs(cuda_device):
    """Run each full-size workload once on the GPU and the oracle once on its
    sampled rows; the tests below share the results."""
    cache = {}

    def get(name):
        if name in cache:
            return cache[name]
        w = inputs.WORKLOADS[name]
        X, W, lab = inputs.make_workload(w, device=cuda_device)
        p = flce.make_problem(w.BT, w.H, w.V, X.dtype, softcap=w.softcap)
        ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
        loss, dX, dW = flce.fused(X, W, lab, softcap=w.softcap, ws=ws)
        status, nv = flce.flce_get_device_status(ws)
        loss2, dX2, dW2 = flce.fused(X, W, lab, softcap=w.softcap, ws=ws)
        same = (loss2.item() == loss.item() and torch.equal(dX2, dX) and torch.equal(dW2, dW))
        del dX2, dW2, ws
        loss_f, lse = flce.forward(X, W, lab, softcap=w.softcap)
        R = inputs.sample_rows(w.BT, N_ROWS, seed=5)
        Ri = torch.tensor(R, device=cuda_device)
        labc = lab.cpu()
        n_global = oracle.count_valid(labc.numpy())
        o = run_oracle(X[Ri].cpu(), W.cpu(), labc[R], softcap=w.softcap, n_valid=n_global)
        torch.cuda.synchronize()
        res = dict(w=w, X=X, W=W, lab=lab, R=R, Ri=Ri, loss=loss.item(), loss_f=loss_f.item(),
                   status=status, nv=nv, n_global=n_global, same=same, o=o,
                   dX_rows=to_np(dX[Ri]), lse_rows=to_np(lse[Ri]),
                   dW_colsum=dW.float().sum(0).double().cpu().numpy(),
                   dW_colnorm=dW.float().norm(dim=0).double().cpu().numpy(),
                   finite=bool(torch.isfinite(dX).all() and torch.isfinite(dW).all()))
        del dX, dW
        cache[name] = res
        return res

    return get


@pytest.mark.parametrize("name", FULL)
def test_full_size_rows_and_invariants(name, full_runs):
    r = full_runs(name)
    w, o, tol = r["w"], r["o"], TOL["bf16"]
    assert r["status"] == 0
    assert r["nv"] == r["n_global"]                       # exact
    assert r["finite"]
    assert r["same"]                                      # bitwise deterministic
    assert rel_scalar(r["loss"], r["loss_f"]) <= tol["loss"]
    lse_err = np.max(np.abs(r["lse_rows"] - o["lse"]) / np.maximum(1.0, np.abs(o["lse"])))
    assert lse_err <= tol["lse"], lse_err
    assert rel_fro(r["dX_rows"], o["dX"]) <= tol["grad"]
    if w.softcap == 0:
        ratio = np.abs(r["dW_colsum"]) / np.maximum(r["dW_colnorm"], 1e-30)
        assert np.max(ratio) <= 2e-2, np.max(ratio)


@pytest.mark.parametrize("sched", ["recompute", "fused_fwd"])
@pytest.mark.parametrize("name", FULL)
def test_full_width_row_subset(name, sched, full_runs):
    """The sampled rows as a problem of their own (full V and H): with dloss =
    N_rows / N_global its gradients are the oracle's for those rows with the
    global mean, so loss, dX and the whole V x H dW can be compared."""
    r = full_runs(name)
    w, o, tol = r["w"], r["o"], TOL["bf16"]
    Xs = r["X"][r["Ri"]].contiguous()
    ls = r["lab"][r["Ri"]].contiguous()
    n_rows = int((ls != inputs.IGNORE_INDEX).sum().item())
    which = {"recompute": flce.FLCE_SCHEDULE_RECOMPUTE,
             "fused_fwd": flce.FLCE_SCHEDULE_FUSED_FORWARD}[sched]
    with _Schedule(which):
        loss, dX, dW = flce.fused(Xs, r["W"], ls, softcap=w.softcap,
                                  dloss=n_rows / r["n_global"])
    torch.cuda.synchronize()
    assert rel_scalar(loss.item() * n_rows / r["n_global"], o["loss"]) <= tol["loss"]
    assert rel_fro(to_np(dX), o["dX"]) <= tol["grad"]
    assert rel_fro(to_np(dW), o["dW"]) <= tol["grad"]


RAGGED = [0, 5, 81]  # BT = 4096, a ragged value, 32768


@pytest.mark.parametrize("idx", RAGGED)
def test_ragged_bt_sweep_rows(idx, cuda_device):
    bts = inputs.ragged_bt_list()
    w = inputs.ragged_workload(idx, bts[idx])
    X, W, lab = inputs.make_workload(w, device=cuda_device)
    p = flce.make_problem(w.BT, w.H, w.V, X.dtype)
    ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
    loss, dX, dW = flce.fused(X, W, lab, ws=ws)
    status, nv = flce.flce_get_device_status(ws)
    labc = lab.cpu()
    assert status == 0 and nv == oracle.count_valid(labc.numpy())
    R = inputs.sample_rows(w.BT, 8, seed=idx)
    Ri = torch.tensor(R, device=cuda_device)
    o = run_oracle(X[Ri].cpu(), W.cpu(), labc[R], n_valid=nv, want_dW=False)
    assert rel_fro(to_np(dX[Ri]), o["dX"]) <= TOL["bf16"]["grad"]
    assert bool(torch.isfinite(dW).all())


def _pairs_problem(w, D, seed, device):
    """A full-size problem whose BT rows are D distinct (hidden state, label)
    pairs, pair d repeated count_d times and scattered by a seeded
    permutation over every row chunk.  Counts come in four classes of D/4
    pairs with unequal multiplicities.  Returns the distinct pairs, the class
    of each pair, the class counts and the row -> pair index."""
    Xd, W, labd = inputs.make_workload(w, device=device, BT=D)
    labd = labd.clone()
    if w.ignore_frac > 0:
        labd[[3, 22, 41]] = inputs.IGNORE_INDEX      # ignored pairs in three classes
    base = w.BT // D
    counts = [base * 4 // 10, base * 7 // 10, base * 12 // 10]
    counts.append(4 * base - sum(counts))            # the classes together fill BT
    per_class = D // 4
    cls = np.repeat(np.arange(4), per_class)
    mult = np.array([counts[c] for c in cls])
    assert mult.sum() == w.BT and len(set(counts)) == 4
    g = torch.Generator().manual_seed(seed)
    idx = torch.repeat_interleave(torch.arange(D), torch.tensor(mult))
    idx = idx[torch.randperm(w.BT, generator=g)]
    return Xd, W, labd, cls, counts, idx


@pytest.mark.parametrize("name", FULL)
def test_full_size_dW_vs_oracle(name, cuda_device):
    """The whole V x H dW and BT x H dX of a full-size call (automatic
    schedule, the bench's launch configuration, every row chunk, the fp32
    running sum read back) against the oracle element by element.  With the
    rows built from D distinct pairs, dW = sum_d count_d G_d^T x_d: the oracle
    runs each multiplicity class's pairs once (global N_valid) and the class
    dW's are weighted by the class count, in fp64."""
    w = inputs.WORKLOADS[name]
    D = 64
    Xd, W, labd, cls, counts, idx = _pairs_problem(w, D, seed=17, device=cuda_device)
    idx_d = idx.to(cuda_device)
    X = Xd[idx_d].contiguous()
    lab = labd[idx_d].contiguous()
    p = flce.make_problem(w.BT, w.H, w.V, X.dtype, softcap=w.softcap)
    ws = flce.workspace(p, flce.FLCE_OP_FUSED, cuda_device)
    loss, dX, dW = flce.fused(X, W, lab, softcap=w.softcap, ws=ws)
    status, nv = flce.flce_get_device_status(ws)
    labc = labd.cpu()
    valid = (labc != inputs.IGNORE_INDEX).numpy()
    n_global = int(sum(counts[c] for c, v in zip(cls, valid) if v))
    assert status == 0 and nv == n_global == oracle.count_valid(lab.cpu().numpy())
    del ws
    Xc, Wc = Xd.cpu(), W.cpu()
    dW_ref = None
    dX_pairs = np.zeros((D, w.H))
    loss_ref = 0.0
    for c in range(4):
        rows = np.nonzero(cls == c)[0]
        o = run_oracle(Xc[rows], Wc, labc[rows], softcap=w.softcap, n_valid=n_global)
        dX_pairs[rows] = o["dX"]
        loss_ref += counts[c] * o["loss"]
        o["dW"] *= counts[c]
        if dW_ref is None:
            dW_ref = o["dW"]
        else:
            dW_ref += o["dW"]
        del o
    tol = TOL["bf16"]
    assert rel_scalar(loss.item(), loss_ref) <= tol["loss"]
    # dX: every row against its pair's oracle row
    dX_ref = torch.from_numpy(dX_pairs).to(cuda_device)[idx_d]
    err = float((dX.double() - dX_ref).norm() / dX_ref.norm())
    assert err <= tol["grad"], err
    del dX_ref
    # dW: the whole matrix, compared in row blocks on the GPU
    num = den = 0.0
    for r0 in range(0, w.V, 16384):
        ref = torch.from_numpy(dW_ref[r0:r0 + 16384]).to(cuda_device)
        num += float(((dW[r0:r0 + 16384].double() - ref) ** 2).sum())
        den += float((ref ** 2).sum())
    assert (num / den) ** 0.5 <= tol["grad"], (num / den) ** 0.5
