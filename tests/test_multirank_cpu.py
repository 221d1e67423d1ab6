"""bench.py's multi-rank plumbing on CPU with gloo, world size 2: the job's
time is the slowest rank's, barriers pair up, and ranks agree."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + rank * 2.5, world)
        bench.barrier(world)
        q.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 12.5, 1: 12.5}


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def _ref_step(X, W, lab, n):
    """fp64 torch restatement of one rank's share (test-only): the mean is
    over n rows, the rank's loss and dW are its shares."""
    z = X @ W.T
    lse = torch.logsumexp(z, dim=1)
    valid = lab != -100
    safe = torch.where(valid, lab, torch.zeros_like(lab))
    nn = float(n.item())
    nll = torch.where(valid, lse - z[torch.arange(z.shape[0]), safe], torch.zeros_like(lse))
    loss = (nll.sum() / nn if nn > 0 else nll.sum() * 0).reshape(1)
    G = torch.softmax(z, dim=1)
    G[torch.arange(z.shape[0]), safe] -= 1.0
    G = G * valid[:, None] / (nn if nn > 0 else 1.0)
    return loss, G @ W, G.T @ X


def _dp_worker(rank, world, port, q, shards):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_cross_entropy_tiles_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        X, W, lab = shards[rank]
        loss, dX, dW, n = dp.data_parallel_step(
            lambda: (lab != -100).sum().reshape(1).to(torch.int64),
            lambda n: _ref_step(X, W, lab, n))
        # numpy copies: a tensor on the queue would be shared memory that this
        # process releases when it exits
        q.put((rank, loss.numpy().copy(), dX.numpy().copy(), dW.numpy().copy(), int(n.item())))
    finally:
        dist.destroy_process_group()


def test_data_parallel_step_gloo_world2():
    """Rows split unevenly over two ranks (one rank's rows all ignored in the
    second case): the global N_valid, the summed loss shares and the summed
    dW equal the single-process result over all rows; each rank's dX equals
    those rows of the full dX."""
    g = torch.Generator().manual_seed(7)
    H, V = 16, 37
    for ignored_rank1 in (False, True):
        X = torch.randn(12, H, generator=g, dtype=torch.float64)
        W = 0.3 * torch.randn(V, H, generator=g, dtype=torch.float64)
        lab = torch.randint(0, V, (12,), generator=g)
        lab[2] = -100
        if ignored_rank1:
            lab[5:] = -100
        shards = [(X[:5], W, lab[:5]), (X[5:], W, lab[5:])]
        n_all = torch.tensor([int((lab != -100).sum())])
        ref_loss, ref_dX, ref_dW = _ref_step(X, W, lab, n_all)
        ctx = mp.get_context("spawn")
        q = ctx.Queue()
        port = _free_port()
        procs = [ctx.Process(target=_dp_worker, args=(r, 2, port, q, shards)) for r in range(2)]
        for p in procs:
            p.start()
        got = {}
        for _ in range(2):
            r, loss, dX, dW, n = q.get(timeout=120)
            got[r] = (loss, dX, dW, n)
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        for r, rows in ((0, slice(0, 5)), (1, slice(5, 12))):
            loss, dX, dW, n = (torch.from_numpy(got[r][0]), torch.from_numpy(got[r][1]),
                               torch.from_numpy(got[r][2]), got[r][3])
            assert n == int(n_all.item())
            assert torch.allclose(loss, ref_loss, rtol=1e-12, atol=1e-14)
            assert torch.allclose(dW, ref_dW, rtol=1e-12, atol=1e-14)
            assert torch.allclose(dX, ref_dX[rows], rtol=1e-12, atol=1e-14)


def _sliced_worker(rank, world, port, q, shards, bounds, shard):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_cross_entropy_tiles_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        X, W, lab = shards[rank]

        def compute(n, events):
            assert events is None  # CPU tensors: final when compute returns
            return _ref_step(X, W, lab, n)

        loss, dX, dW, n = dp.data_parallel_step_sliced(
            lambda: (lab != -100).sum().reshape(1).to(torch.int64), compute, bounds,
            shard=shard)
        q.put((rank, loss.numpy().copy(), dX.numpy().copy(), dW.numpy().copy(), int(n.item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shard", [(2, False), (3, False), (2, True), (3, True)])
def test_sliced_dW_exchange_gloo(world, shard):
    """The overlapped exchange of flce_fused_global_sliced's dW: slices of
    whole 256-row tiles (here 4-row pieces of a 37-row dW, trailing slices
    empty), each all-reduced, or reduced onto its rank (reduce-scatter):
    every rank gets the summed dW, or exactly its own rows of it."""
    g = torch.Generator().manual_seed(11)
    H, V, BT = 8, 37, 14
    X = torch.randn(BT, H, generator=g, dtype=torch.float64)
    W = 0.3 * torch.randn(V, H, generator=g, dtype=torch.float64)
    lab = torch.randint(0, V, (BT,), generator=g)
    lab[[1, 9]] = -100
    cuts = [0, 4, 9, BT][:world] + [BT]
    shards = [(X[cuts[r]:cuts[r + 1]], W, lab[cuts[r]:cuts[r + 1]]) for r in range(world)]
    n_all = torch.tensor([int((lab != -100).sum())])
    ref_loss, ref_dX, ref_dW = _ref_step(X, W, lab, n_all)
    if shard:
        r = 16  # rows per slice; the third rank's slice is empty when world = 3
        bounds = [(min(V, s * r), min(V, (s + 1) * r)) for s in range(world)]
    else:
        bounds = [(0, 12), (12, 24), (24, 37), (37, 37)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sliced_worker, args=(r, world, port, q, shards, bounds, shard))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, rest) for r, *rest in (q.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    for r in range(world):
        loss, dX, dW, n = got[r]
        assert n == int(n_all.item())
        assert torch.allclose(torch.from_numpy(loss), ref_loss, rtol=1e-12, atol=1e-14)
        assert torch.allclose(torch.from_numpy(dX), ref_dX[cuts[r]:cuts[r + 1]], rtol=1e-12,
                              atol=1e-14)
        want = ref_dW[bounds[r][0]:bounds[r][1]] if shard else ref_dW
        assert tuple(dW.shape) == tuple(want.shape)
        assert torch.allclose(torch.from_numpy(dW), want, rtol=1e-12, atol=1e-14)


def _dw_reduce_worker(rank, world, port, q, shares):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_cross_entropy_tiles_b200 import dp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out = {}
        for dt in (torch.float32, torch.bfloat16):
            share = shares[rank].to(dt)
            _, _, dW, _ = dp.data_parallel_step(
                lambda: torch.ones(1, dtype=torch.int64),
                lambda n: (torch.zeros(1), torch.zeros(1), share.clone()))
            out[str(dt)] = dW.float().numpy().copy()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_dw_summed_over_ranks_in_fp32(world):
    """Each rank's dW share in fp32 (what dp.fused_dp has the library write)
    summed by the collective in fp32: every rank gets the same sum, within
    fp32 rounding of the exact (fp64) sum of the shares.  The same shares
    rounded to bf16 and summed in bf16 are off by bf16's 8-bit rounding,
    hundreds of times more: why the fp32 reduction is the default."""
    g = torch.Generator().manual_seed(11)
    shares = [torch.randn(64, 48, generator=g, dtype=torch.float64) * 1e-3
              for _ in range(world)]
    exact = sum(shares)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dw_reduce_worker, args=(r, world, port, q, shares))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    ref = exact.numpy()
    scale = float(abs(ref).max())
    f32 = [got[r]["torch.float32"] for r in range(world)]
    b16 = [got[r]["torch.bfloat16"] for r in range(world)]
    assert all((f == f32[0]).all() for f in f32) and all((b == b16[0]).all() for b in b16)
    err32 = float(abs(f32[0] - ref).max()) / scale
    err16 = float(abs(b16[0] - ref).max()) / scale
    assert err32 <= world * 2.0 ** -23
    assert err16 >= 100 * err32 and err16 <= world * 2.0 ** -8


def _vp_ref_stats(X, W_r, lab, v_off):
    """fp64 torch restatement (test-only) of one rank's slice statistics."""
    z = X @ W_r.T
    u = z * 1.4426950408889634
    m = u.max(dim=1).values
    s = torch.exp2(u - m[:, None]).sum(1)
    here = (lab >= v_off) & (lab < v_off + W_r.shape[0]) & (lab != -100)
    idx = torch.where(here, lab - v_off, torch.zeros_like(lab))
    tgt = torch.where(here, z[torch.arange(z.shape[0]), idx], torch.zeros_like(m))
    return torch.stack([m, s, tgt], 1)


def _vp_ref_combine(stats_all, lab):
    M = stats_all[:, :, 0].max(0).values
    S = (stats_all[:, :, 1] * torch.exp2(stats_all[:, :, 0] - M)).sum(0)
    lse = (M + torch.log2(S)) * 0.6931471805599453
    valid = lab != -100
    n = int(valid.sum())
    nll = torch.where(valid, lse - stats_all[:, :, 2].sum(0), torch.zeros_like(lse))
    return (nll.sum() / max(n, 1)).reshape(1), lse


def _vp_ref_backward(X, W_r, lab, v_off, lse):
    z = X @ W_r.T
    G = torch.exp(z - lse[:, None])
    here = (lab >= v_off) & (lab < v_off + W_r.shape[0]) & (lab != -100)
    rows = torch.nonzero(here).flatten()
    G[rows, lab[rows] - v_off] -= 1.0
    valid = lab != -100
    n = int(valid.sum())
    G = G * valid[:, None] / max(n, 1)
    return G @ W_r, G.T @ X


def _vp_worker(rank, world, port, q, X, W, lab, slices):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from linear_cross_entropy_tiles_b200 import vp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        off, n = slices[rank]
        W_r = W[off:off + n]
        loss, lse, dX, dW = vp.vocab_parallel_step(
            lambda: _vp_ref_stats(X, W_r, lab, off),
            lambda st: _vp_ref_combine(st, lab),
            lambda l: _vp_ref_backward(X, W_r, lab, off, l))
        q.put((rank, loss.numpy().copy(), lse.numpy().copy(), dX.numpy().copy(),
               dW.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_parallel_step_gloo(world):
    """W split over the vocabulary in uneven slices: the gathered slice
    statistics give every rank the single-process lse and loss; the summed dX
    shares give the full dX; each rank's dW is its rows of the full dW.
    Labels fall in every slice, one row is ignored."""
    from linear_cross_entropy_tiles_b200 import vp
    g = torch.Generator().manual_seed(21)
    BT, H, V = 10, 8, 23
    X = torch.randn(BT, H, generator=g, dtype=torch.float64)
    W = 0.7 * torch.randn(V, H, generator=g, dtype=torch.float64)
    lab = torch.randint(0, V, (BT,), generator=g)
    lab[3] = -100
    slices = vp.vp_offsets(V, world)
    assert sum(n for _, n in slices) == V and len({n for _, n in slices}) <= 2
    z = X @ W.T
    lse_ref = torch.logsumexp(z, 1)
    G = torch.softmax(z, 1)
    valid = lab != -100
    G[valid.nonzero().flatten(), lab[valid]] -= 1.0
    G = G * valid[:, None] / int(valid.sum())
    loss_ref = (lse_ref - z[torch.arange(BT), lab.clamp(min=0)])[valid].mean()
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_vp_worker, args=(r, world, port, qq, X, W, lab, slices))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, rest) for r, *rest in (qq.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    for r, (off, n) in enumerate(slices):
        loss, lse, dX, dW = (torch.from_numpy(a) for a in got[r])
        assert torch.allclose(loss, loss_ref.reshape(1), rtol=1e-12)
        assert torch.allclose(lse, lse_ref, rtol=1e-12)
        assert torch.allclose(dX, G @ W, rtol=1e-10, atol=1e-14)
        assert torch.allclose(dW, (G.T @ X)[off:off + n], rtol=1e-10, atol=1e-14)
