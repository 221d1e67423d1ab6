"""Cross-entropy from logits the caller holds (flce_ce_forward /
flce_ce_backward) against the oracle's ``ce``, element by element.

PyTorch PR #126348's case: the forward reads the logits once and keeps
lse; the backward reads them again and rebuilds the softmax from them and
lse (point b.).  Small problems cover rows that do not start on a 16-byte
boundary (odd V), V below one 16-byte vector, row strides whose input and
output rows differ in alignment, the in-place gradient, the in-op label
shift, ignored rows, the softcap, -inf and huge logits; the llm.c shape of
the PR (32 x 1024 rows, V = 50257, bf16) is checked at full size."""
import numpy as np
import pytest
import torch

import linear_cross_entropy_tiles_b200 as flce
import oracle
from linear_cross_entropy_tiles_b200 import inputs
from parity import TOL, rel_fro, rel_scalar, to_np

pytestmark = pytest.mark.gpu

IGN = inputs.IGNORE_INDEX


def _logits(BT, V, dtype, std, seed, ignore_frac=0.0):
    g = torch.Generator().manual_seed(seed)
    Z = (torch.randn(BT, V, generator=g) * std).to(inputs.torch_dtype(dtype))
    lab = torch.randint(0, V, (BT,), generator=g, dtype=torch.int64)
    n = int(round(ignore_frac * BT))
    if n:
        lab[torch.randperm(BT, generator=g)[:n]] = IGN
    return Z, lab


def _oracle(Z, lab, **kw):
    za, tag = inputs.oracle_view(Z)
    return oracle.ce(za, lab.numpy(), dtype=tag, **kw)


def _check(o, loss, lse, dZ, dtype, dZ_rows=None):
    tol = TOL[dtype]
    assert rel_scalar(loss, o["loss"]) <= tol["loss"], (loss, o["loss"])
    lse_err = np.max(np.abs(to_np(lse) - o["lse"]) / np.maximum(1.0, np.abs(o["lse"])),
                     initial=0.0)
    assert lse_err <= tol["lse"], lse_err
    if dZ is not None:
        assert rel_fro(to_np(dZ), o["dZ"]) <= tol["grad"]


CASES = [
    # BT, V, dtype, std, softcap, ignore_frac, seed
    (300, 1000, "bf16", 2.0, 0.0, 0.1, 1),
    (129, 50257, "bf16", 3.0, 0.0, 0.05, 2),     # odd V: rows at every 2-byte phase
    (77, 3, "bf16", 1.0, 0.0, 0.0, 3),           # V below one vector
    (33, 9, "bf16", 1.0, 0.0, 0.2, 4),
    (1, 1, "bf16", 1.0, 0.0, 0.0, 5),
    (257, 20000, "bf16", 8.0, 30.0, 0.1, 6),     # softcap
    (64, 513, "fp32", 2.0, 0.0, 0.1, 7),
    (100, 7777, "fp32", 4.0, 5.0, 0.1, 8),
    (40, 130001, "bf16", 2.0, 0.0, 0.0, 9),      # long rows
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%d-%s-cap%g" % (c[0], c[1], c[2], c[4]))
def test_ce_forward_backward_match_oracle(case, cuda_device):
    BT, V, dtype, std, cap, ign, seed = case
    Z, lab = _logits(BT, V, dtype, std, seed, ign)
    o = _oracle(Z, lab, softcap=cap, dloss=0.75)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    p = flce.make_ce_problem(BT, V, Zd.dtype, softcap=cap)
    ws = flce.ce_workspace(p, flce.FLCE_OP_FORWARD, cuda_device)
    loss, lse = flce.ce_forward(Zd, labd, softcap=cap, ws=ws)
    st, nv = flce.flce_get_device_status(ws)
    assert st == 0 and nv == o["n_valid"]               # ignore mask: exact
    dl = torch.tensor([0.75], device=cuda_device)
    dZ = flce.ce_backward(Zd, labd, lse, dl, softcap=cap)
    torch.cuda.synchronize()
    _check(o, loss.item(), lse, dZ, dtype)
    # ignored rows: exactly zero gradient
    ign_rows = (lab == IGN).nonzero().flatten().tolist()
    if ign_rows:
        assert not dZ[ign_rows].any()
    # bitwise deterministic
    loss2, lse2 = flce.ce_forward(Zd, labd, softcap=cap)
    assert loss2.item() == loss.item() and torch.equal(lse2, lse)
    assert torch.equal(flce.ce_backward(Zd, labd, lse, dl, softcap=cap), dZ)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("pad_in,pad_out", [(3, 0), (0, 5), (8, 16), (1, 1)])
def test_ce_row_strides(dtype, pad_in, pad_out, cuda_device):
    """Logits as a column slice [:, :V] of a [BT, V + pad_in] buffer and the
    gradient into a slice of a [BT, V + pad_out] buffer: the input and output
    rows start at different 16-byte phases when the pads differ.  Where the
    input rows keep the dense run's phases (pad_in a multiple of 16 bytes)
    the sums run in the same order and the results are equal bit for bit;
    otherwise a row splits into its scalar and vector parts elsewhere, the
    sums are reordered, and lse agrees to fp32 rounding.  The columns past V
    of the gradient buffer are never written."""
    BT, V = 150, 1001
    Z, lab = _logits(BT, V, dtype, 2.0, 11, 0.1)
    dt = inputs.torch_dtype(dtype)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    big = torch.full((BT, V + pad_in), float("nan"), dtype=dt, device=cuda_device)
    big[:, :V] = Zd
    out_big = torch.full((BT, V + pad_out), 7.0, dtype=dt, device=cuda_device)
    loss_a, lse_a = flce.ce_forward(Zd, labd)
    loss_b, lse_b = flce.ce_forward(big[:, :V], labd)
    dl = torch.tensor([1.0], device=cuda_device)
    dZ_a = flce.ce_backward(Zd, labd, lse_a, dl)
    dZ_b = flce.ce_backward(big[:, :V], labd, lse_b, dl, out=out_big[:, :V])
    torch.cuda.synchronize()
    if (pad_in * Zd.element_size()) % 16 == 0:
        assert loss_a.item() == loss_b.item() and torch.equal(lse_a, lse_b)
        assert torch.equal(dZ_a, dZ_b)
    else:
        assert float(((lse_a - lse_b).abs() / lse_a.abs()).max()) <= 1e-6
        assert rel_fro(to_np(dZ_b), to_np(dZ_a)) <= (1e-5 if dtype == "fp32" else 4e-3)
    if pad_out:
        assert bool((out_big[:, V:] == 7.0).all())
    o = _oracle(Z, lab)
    _check(o, loss_a.item(), lse_a, dZ_a, dtype)


def test_ce_in_place_gradient(cuda_device):
    """dlogits == logits: the gradient overwrites the logits, equal to the
    out-of-place result bit for bit."""
    BT, V = 200, 4099
    Z, lab = _logits(BT, V, "bf16", 3.0, 12, 0.1)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    loss, lse = flce.ce_forward(Zd, labd, softcap=20.0)
    dl = torch.tensor([2.0], device=cuda_device)
    ref = flce.ce_backward(Zd, labd, lse, dl, softcap=20.0)
    Zi = Zd.clone()
    out = flce.ce_backward(Zi, labd, lse, dl, softcap=20.0, out=Zi)
    torch.cuda.synchronize()
    assert out.data_ptr() == Zi.data_ptr() and torch.equal(Zi, ref)


@pytest.mark.parametrize("B,T", [(4, 100), (3, 1)])
def test_ce_in_op_label_shift(B, T, cuda_device):
    """shift_seq_len = T: the caller passes the full (B*T, V) logits and the
    (B, T) token ids, with no logits[..., :-1, :] / labels[..., 1:] copies."""
    V = 777
    Z, ids = _logits(B * T, V, "bf16", 2.0, 13)
    lab = torch.cat([ids.reshape(B, T)[:, 1:], torch.full((B, 1), IGN, dtype=ids.dtype)],
                    1).reshape(-1)
    Zd, idsd = Z.to(cuda_device), ids.to(cuda_device)
    p = flce.make_ce_problem(B * T, V, Zd.dtype, shift_seq_len=T)
    ws = flce.ce_workspace(p, flce.FLCE_OP_FORWARD, cuda_device)
    loss, lse = flce.ce_forward(Zd, idsd, ws=ws, shift_seq_len=T)
    st, nv = flce.flce_get_device_status(ws)
    dl = torch.tensor([1.0], device=cuda_device)
    dZ = flce.ce_backward(Zd, idsd, lse, dl, shift_seq_len=T)
    torch.cuda.synchronize()
    assert st == 0 and nv == oracle.count_valid(lab.numpy())
    if nv == 0:
        assert loss.item() == 0.0 and not dZ.any()
        return
    _check(_oracle(Z, lab), loss.item(), lse, dZ, "bf16")


def test_ce_all_ignored_empty_and_bad_label(cuda_device):
    Z, lab = _logits(50, 300, "bf16", 1.0, 14)
    Zd = Z.to(cuda_device)
    labd = torch.full((50,), IGN, dtype=torch.int64, device=cuda_device)
    loss, lse = flce.ce_forward(Zd, labd)
    dZ = flce.ce_backward(Zd, labd, lse, torch.ones(1, device=cuda_device))
    assert loss.item() == 0.0 and not dZ.any()
    # empty batch
    E = torch.empty(0, 300, dtype=torch.bfloat16, device=cuda_device)
    el = torch.empty(0, dtype=torch.int64, device=cuda_device)
    loss, lse = flce.ce_forward(E, el)
    assert loss.item() == 0.0 and lse.numel() == 0
    assert flce.ce_backward(E, el, lse, torch.ones(1, device=cuda_device)).numel() == 0
    # a label outside [0, V): reported on the device, the next call is clean
    labd = lab.to(cuda_device)
    labd[17] = 300
    p = flce.make_ce_problem(50, 300, Zd.dtype)
    ws = flce.ce_workspace(p, flce.FLCE_OP_FORWARD, cuda_device)
    loss = torch.empty(1, device=cuda_device)
    lse = torch.empty(50, device=cuda_device)
    flce.flce_ce_forward(p, Zd, labd, loss, lse, ws)
    assert flce.flce_get_device_status(ws)[0] == 5
    labd[17] = 0
    flce.flce_ce_forward(p, Zd, labd, loss, lse, ws)
    assert flce.flce_get_device_status(ws)[0] == 0


def test_ce_extreme_logits(cuda_device):
    """Logits near +-1000 and -inf entries (a masked vocabulary): the online
    max keeps every sum finite, -inf entries get probability and gradient 0."""
    BT, V = 64, 2000
    Z, lab = _logits(BT, V, "fp32", 1.0, 15)
    Z[:8] += 1000.0
    Z[8:16] -= 1000.0
    Z[16:32, 100:400] = float("-inf")
    lab[16:32] = 5
    o = _oracle(Z, lab)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    loss, lse = flce.ce_forward(Zd, labd)
    dZ = flce.ce_backward(Zd, labd, lse, torch.ones(1, device=cuda_device))
    torch.cuda.synchronize()
    assert torch.isfinite(dZ).all() and torch.isfinite(lse).all()
    assert not dZ[16:32, 100:400].any()
    _check(o, loss.item(), lse, dZ, "fp32")


def test_ce_llmc_shape_full_size(cuda_device):
    """PR #126348's llm.c tensor: B=32, T=1024, V=50257, bf16 (about 3.3 GB of
    logits), the launch configuration bench.py times.  The loss and every
    row's lse are compared with the oracle over all rows, the gradient on
    512 sampled rows (rows are independent given the global N_valid), plus
    invariants of the whole gradient: each valid row sums to ~0, ignored
    rows are 0."""
    w = inputs.CE_WORKLOADS["ce_llmc"]
    Z, lab = inputs.make_ce_workload(w, device=cuda_device)
    loss, lse = flce.ce_forward(Z, lab)
    dZ = flce.ce_backward(Z, lab, lse, torch.ones(1, device=cuda_device))
    torch.cuda.synchronize()
    Zc, labc = Z.cpu(), lab.cpu()
    o_all = _oracle(Zc, labc, grads=False)
    _check(o_all, loss.item(), lse, None, "bf16")
    R = inputs.sample_rows(w.BT, 512, seed=3)
    o = _oracle(Zc[R], labc[R], n_valid=o_all["n_valid"])
    assert rel_fro(to_np(dZ[R]), o["dZ"]) <= TOL["bf16"]["grad"]
    row_sum = dZ.float().sum(1)
    row_abs = dZ.float().abs().sum(1)
    assert float((row_sum.abs() / row_abs.clamp_min(1e-30)).max()) <= 2e-2


FUSED_CASES = CASES + [(8, 60000, "fp32", 3.0, 0.0, 0.0, 31),   # fp32 row > 112 KB: L2 path
                       (16, 130001, "bf16", 3.0, 20.0, 0.1, 32),
                       # many rows per block: both row buffers reused many times
                       (1500, 3001, "bf16", 2.0, 10.0, 0.1, 33),
                       (2000, 700, "fp32", 3.0, 0.0, 0.05, 34)]


@pytest.mark.parametrize("case", FUSED_CASES,
                         ids=lambda c: "%dx%d-%s-cap%g" % (c[0], c[1], c[2], c[4]))
def test_ce_fused_matches_oracle_and_the_two_calls(case, cuda_device):
    """flce_ce_fused (each row read once into shared memory, or re-read
    from L2 for rows over 112 KB) against the oracle, and against the
    forward + backward pair to fp32 rounding (their sums run in another
    order)."""
    BT, V, dtype, std, cap, ign, seed = case
    Z, lab = _logits(BT, V, dtype, std, seed, ign)
    o = _oracle(Z, lab, softcap=cap, dloss=0.75)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    loss, lse, dZ = flce.ce_fused(Zd, labd, softcap=cap, dloss=0.75)
    loss2, lse2 = flce.ce_forward(Zd, labd, softcap=cap)
    dZ2 = flce.ce_backward(Zd, labd, lse2, torch.tensor([0.75], device=cuda_device), softcap=cap)
    torch.cuda.synchronize()
    _check(o, loss.item(), lse, dZ, dtype)
    assert float(((lse - lse2).abs() / lse2.abs().clamp_min(1.0)).max()) <= 1e-6
    assert rel_fro(to_np(dZ), to_np(dZ2)) <= (1e-5 if dtype == "fp32" else 4e-3)
    ign_rows = (lab == IGN).nonzero().flatten().tolist()
    if ign_rows:
        assert not dZ[ign_rows].any()
    l3, _, dZ3 = flce.ce_fused(Zd, labd, softcap=cap, dloss=0.75, want_lse=False)
    assert l3.item() == loss.item() and torch.equal(dZ3, dZ)     # deterministic, lse optional


@pytest.mark.parametrize("pad_out", [0, 3])
def test_ce_fused_in_place_and_strided(pad_out, cuda_device):
    BT, V = 130, 5003
    Z, lab = _logits(BT, V, "bf16", 2.0, 33, 0.1)
    Zd, labd = Z.to(cuda_device), lab.to(cuda_device)
    ref = flce.ce_fused(Zd, labd, softcap=15.0)
    if pad_out == 0:                       # in place
        Zi = Zd.clone()
        out = flce.ce_fused(Zi, labd, softcap=15.0, out=Zi)
        assert out[2].data_ptr() == Zi.data_ptr()
    else:                                  # output rows at another 16-byte phase
        big = torch.full((BT, V + pad_out), 7.0, dtype=Zd.dtype, device=cuda_device)
        out = flce.ce_fused(Zd, labd, softcap=15.0, out=big[:, :V])
        assert bool((big[:, V:] == 7.0).all())
    torch.cuda.synchronize()
    assert out[0].item() == ref[0].item() and torch.equal(out[2], ref[2])


def test_ce_fused_shift_and_llmc_full_size(cuda_device):
    B, T, V = 3, 200, 1000
    Z, ids = _logits(B * T, V, "bf16", 2.0, 34)
    lab = torch.cat([ids.reshape(B, T)[:, 1:], torch.full((B, 1), IGN, dtype=ids.dtype)],
                    1).reshape(-1)
    loss, lse, dZ = flce.ce_fused(Z.to(cuda_device), ids.to(cuda_device), shift_seq_len=T)
    _check(_oracle(Z, lab), loss.item(), lse, dZ, "bf16")
    # the llm.c tensor: all rows' lse and the loss against the oracle, 512
    # sampled gradient rows
    w = inputs.CE_WORKLOADS["ce_llmc"]
    Zf, labf = inputs.make_ce_workload(w, device=cuda_device)
    loss, lse, dZ = flce.ce_fused(Zf, labf)
    torch.cuda.synchronize()
    Zc, labc = Zf.cpu(), labf.cpu()
    o_all = _oracle(Zc, labc, grads=False)
    _check(o_all, loss.item(), lse, None, "bf16")
    R = inputs.sample_rows(w.BT, 512, seed=4)
    o = _oracle(Zc[R], labc[R], n_valid=o_all["n_valid"])
    assert rel_fro(to_np(dZ[R]), o["dZ"]) <= TOL["bf16"]["grad"]
