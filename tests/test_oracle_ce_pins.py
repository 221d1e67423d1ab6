"""Pins for the oracle's cross-entropy-from-logits function (``oracle.ce``),
the case of PyTorch PR #126348: the caller holds softmax_input, the forward
keeps only the per-row max/sum (steps 2-3) and the label's entry (point a.),
and the backward rebuilds the softmax from the logits (point b.).

Each pin checks the oracle against something the mathematics fixes, not
against its own formula retyped: exact closed forms, invariances of the
softmax, central finite differences, an independent library routine (torch
fp64 cross_entropy + autograd), and the FLCE oracle on logits a separate
numpy matmul produced."""
import math

import numpy as np
import pytest
import torch

import oracle

IGN = -100


def _rand(BT, V, seed, std=1.5, ignore=()):
    rs = np.random.RandomState(seed)
    Z = rs.randn(BT, V) * std
    lab = rs.randint(0, V, BT).astype(np.int64)
    for i in ignore:
        lab[i] = IGN
    return Z, lab


def test_hand_example_three_classes():
    """Logits (0, ln2, ln5): exps 1, 2, 5, sum 8.  Label 1: loss = ln8 - ln2 =
    ln4, dZ = (1/8, 2/8 - 1, 5/8); an ignored second row adds nothing."""
    Z = np.array([[0.0, math.log(2.0), math.log(5.0)], [3.0, -1.0, 0.5]])
    o = oracle.ce(Z, np.array([1, IGN], np.int64))
    assert o["n_valid"] == 1
    assert o["lse"][0] == pytest.approx(math.log(8.0), rel=1e-15)
    assert o["lse"][1] == pytest.approx(math.log(math.exp(3) + math.exp(-1) + math.exp(0.5)),
                                        rel=1e-15)
    assert o["loss"] == pytest.approx(math.log(4.0), rel=1e-15)
    np.testing.assert_allclose(o["dZ"][0], [1 / 8, 2 / 8 - 1, 5 / 8], rtol=1e-14)
    assert np.all(o["dZ"][1] == 0.0) and math.isnan(o["target"][1])


def test_hand_example_softcap():
    """c = 2 and z = 2 atanh(1/2) give y = 1; z = 0 gives y = 0.  Label 0:
    loss = ln(1 + e); the capped entry's chain factor is 1 - (1/2)^2 = 3/4."""
    c = 2.0
    Z = np.array([[0.0, c * math.atanh(0.5)]])
    o = oracle.ce(Z, np.array([0], np.int64), softcap=c, dloss=2.0)
    assert o["loss"] == pytest.approx(math.log(1 + math.e), rel=1e-14)
    p1 = math.e / (1 + math.e)
    np.testing.assert_allclose(o["dZ"][0], [2.0 * ((1 - p1) - 1.0), 2.0 * p1 * 0.75], rtol=1e-13)


def test_equal_logits_closed_form():
    """Every logit of a row equal to a constant a: lse = a + ln V, loss = ln V,
    dZ_ij = (1/V - [j = label]) dloss / N on valid rows."""
    BT, V, dl = 7, 11, 0.25
    Z = np.repeat(np.linspace(-3, 4, BT)[:, None], V, axis=1)
    lab = np.array([0, 3, IGN, 10, 5, IGN, 1], np.int64)
    o = oracle.ce(Z, lab, dloss=dl)
    N = 5
    np.testing.assert_allclose(o["lse"], Z[:, 0] + math.log(V), rtol=1e-15)
    assert o["loss"] == pytest.approx(math.log(V), rel=1e-14)
    want = np.zeros((BT, V))
    for i in range(BT):
        if lab[i] != IGN:
            want[i] = 1.0 / V
            want[i, lab[i]] -= 1.0
    np.testing.assert_allclose(o["dZ"], want * dl / N, rtol=1e-13, atol=1e-17)


def test_all_ignored_and_empty():
    Z, lab = _rand(5, 9, 1)
    lab[:] = IGN
    o = oracle.ce(Z, lab, softcap=3.0)
    assert o["n_valid"] == 0 and o["loss"] == 0.0 and np.all(o["dZ"] == 0.0)
    o = oracle.ce(np.zeros((0, 9)), np.zeros(0, np.int64))
    assert o["n_valid"] == 0 and o["loss"] == 0.0 and o["dZ"].shape == (0, 9)


def test_bad_labels_rejected():
    Z, lab = _rand(3, 5, 2)
    for bad in (5, -1, 1 << 40):
        lab2 = lab.copy()
        lab2[2] = bad
        with pytest.raises(oracle.OracleLabelError):
            oracle.ce(Z, lab2)


@pytest.mark.parametrize("softcap", [0.0, 3.0, 30.0])
@pytest.mark.parametrize("shape", [(1, 1), (4, 2), (13, 37), (64, 300)])
def test_matches_torch_cross_entropy_autograd(shape, softcap):
    """torch fp64 F.cross_entropy (ignore_index=-100, mean) on the capped
    logits, gradients by autograd: an independent library routine."""
    BT, V = shape
    Z, lab = _rand(BT, V, 3 + BT, std=4.0, ignore=(0,) if BT > 2 else ())
    dl = 0.7
    o = oracle.ce(Z, lab, softcap=softcap, dloss=dl)
    z = torch.tensor(Z, dtype=torch.float64, requires_grad=True)
    y = softcap * torch.tanh(z / softcap) if softcap else z
    valid = int((lab != IGN).sum())
    if valid:
        loss = torch.nn.functional.cross_entropy(y, torch.tensor(lab), ignore_index=IGN)
        (loss * dl).backward()
        assert o["loss"] == pytest.approx(loss.item(), rel=1e-12, abs=1e-14)
        np.testing.assert_allclose(o["dZ"], z.grad.numpy(), rtol=1e-10, atol=1e-14)
    lse = torch.logsumexp(y.detach(), dim=1).numpy()
    np.testing.assert_allclose(o["lse"], lse, rtol=1e-13)


@pytest.mark.parametrize("softcap", [0.0, 2.0])
def test_finite_differences(softcap):
    """Central differences (h = 1e-6) of the loss with respect to every logit."""
    Z, lab = _rand(3, 6, 9, ignore=(1,))
    o = oracle.ce(Z, lab, softcap=softcap, dloss=1.0)
    h = 1e-6
    fd = np.zeros_like(Z)
    for i in range(Z.shape[0]):
        for j in range(Z.shape[1]):
            zp, zm = Z.copy(), Z.copy()
            zp[i, j] += h
            zm[i, j] -= h
            fd[i, j] = (oracle.ce(zp, lab, softcap=softcap, grads=False)["loss"]
                        - oracle.ce(zm, lab, softcap=softcap, grads=False)["loss"]) / (2 * h)
    np.testing.assert_allclose(o["dZ"], fd, rtol=1e-6, atol=1e-9)


def test_shift_invariance_and_zero_row_sums():
    """Without a softcap, adding a constant to a row changes lse by it and
    leaves loss and dZ alone; each valid row of dZ sums to zero."""
    Z, lab = _rand(6, 20, 4, ignore=(2,))
    o = oracle.ce(Z, lab)
    shift = np.arange(6)[:, None] * 7.5 - 10.0
    o2 = oracle.ce(Z + shift, lab)
    np.testing.assert_allclose(o2["lse"], o["lse"] + shift[:, 0], rtol=1e-13)
    assert o2["loss"] == pytest.approx(o["loss"], rel=1e-12)
    np.testing.assert_allclose(o2["dZ"], o["dZ"], rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(o["dZ"].sum(1), 0.0, atol=1e-15)


def test_row_stride_reads_only_the_first_V_columns():
    """Rows ld > V apart: the columns past V are never read (garbage there
    changes nothing) and the result equals the dense V-column problem."""
    Z, lab = _rand(5, 12, 5)
    wide = np.full((5, 20), 1e30)
    wide[:, :12] = Z
    a = oracle.ce(Z, lab, softcap=4.0)
    b = oracle.ce(wide, lab, softcap=4.0, V=12)
    for k in ("lse", "dZ"):
        assert np.array_equal(a[k], b[k])
    assert a["loss"] == b["loss"]


def test_bf16_bits_widen_exactly():
    """bf16 bit patterns give the same result as their exact fp32 values."""
    Z, lab = _rand(4, 33, 6)
    zb = torch.tensor(Z, dtype=torch.float32).to(torch.bfloat16)
    bits = zb.view(torch.int16).numpy().view(np.uint16)
    a = oracle.ce(bits, lab, dtype="bf16")
    b = oracle.ce(zb.float().numpy(), lab)
    assert np.array_equal(a["dZ"], b["dZ"]) and a["loss"] == b["loss"]


@pytest.mark.parametrize("softcap", [0.0, 5.0])
def test_agrees_with_the_flce_oracle_on_matmul_logits(softcap):
    """Logits from a numpy fp64 matmul X W^T fed to oracle.ce reproduce the
    FLCE oracle (its own matmul, loop order and G): lse and loss agree, and
    the chain rule through the matmul turns dZ into the FLCE oracle's dX =
    dZ W and dW = dZ^T X."""
    rs = np.random.RandomState(8)
    BT, H, V = 9, 5, 17
    X = rs.randn(BT, H)
    W = rs.randn(V, H) * 0.8
    lab = rs.randint(0, V, BT).astype(np.int64)
    lab[4] = IGN
    f = oracle.flce(X, W, lab, softcap=softcap, dloss=1.3)
    c = oracle.ce(X @ W.T, lab, softcap=softcap, dloss=1.3)
    np.testing.assert_allclose(c["lse"], f["lse"], rtol=1e-13)
    assert c["loss"] == pytest.approx(f["loss"], rel=1e-13)
    np.testing.assert_allclose(c["dZ"] @ W, f["dX"], rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(c["dZ"].T @ X, f["dW"], rtol=1e-11, atol=1e-15)


def test_global_divisor():
    """A row subset with the global N gives that subset's share: the shares of
    a split sum to the whole problem's loss, and dZ rows are the same."""
    Z, lab = _rand(10, 8, 10, ignore=(3, 7))
    whole = oracle.ce(Z, lab, dloss=1.0)
    N = whole["n_valid"]
    a = oracle.ce(Z[:4], lab[:4], n_valid=N)
    b = oracle.ce(Z[4:], lab[4:], n_valid=N)
    assert a["loss"] + b["loss"] == pytest.approx(whole["loss"], rel=1e-13)
    np.testing.assert_allclose(np.vstack([a["dZ"], b["dZ"]]), whole["dZ"], rtol=1e-14)


def test_huge_logits_stay_finite():
    """Logits near 1000 overflow exp() in fp64 unless the row max is taken
    out first: lse(1000, 990, -1000) = 1000 + ln(1 + e^-10 + e^-2000)."""
    Z = np.array([[1000.0, 990.0, -1000.0], [-5000.0, -5001.0, -5000.0]])
    o = oracle.ce(Z, np.array([1, 2], np.int64))
    assert o["lse"][0] == pytest.approx(1000.0 + math.log1p(math.exp(-10.0)), rel=1e-15)
    assert o["lse"][1] == pytest.approx(-5000.0 + math.log(2.0 + math.exp(-1.0)), rel=1e-15)
    assert np.isfinite(o["dZ"]).all() and math.isfinite(o["loss"])
