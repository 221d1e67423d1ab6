"""The C-ABI library without a GPU: it loads, exports what include/flce.h
declares, sizes workspaces, and rejects bad arguments on the host before any
CUDA call."""
import json
import os
import re

import pytest

import linear_cross_entropy_tiles_b200 as flce
from linear_cross_entropy_tiles_b200 import binding, build, inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    return binding.lib()


def test_exports_every_declared_symbol():
    header = open(os.path.join(ROOT, "include", "flce.h")).read()
    declared = re.findall(r"FLCE_API\s+[\w\s\*]+?\b(flce_\w+)\s*\(", header)
    assert len(declared) == 28
    assert set(declared) == set(binding.EXPORTS)
    lib = binding.lib()
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings():
    for code in range(8):
        assert flce.flce_status_string(code)
    assert "label" in flce.flce_status_string(5)
    assert flce.flce_status_string(99) == "unknown status"


@pytest.mark.parametrize("schedule", [1, 2])
@pytest.mark.parametrize("name", ["gpt2_small", "llama3_8b", "gemma2_softcap", "tiny_fp32"])
def test_workspace_has_no_bt_by_v_buffer(name, schedule):
    """Scratch never scales with BT*V: the recompute schedule stays below one
    BT x V logits tensor; the fused-in-forward one holds at most half of the
    rows' p plus an fp32 V x H running sum of dW and fp32 dX split slabs."""
    w = inputs.WORKLOADS[name]
    dt = flce.FLCE_BF16 if w.dtype == "bf16" else flce.FLCE_FP32
    p = flce.make_problem(w.BT, w.H, w.V, dt, softcap=w.softcap)
    prev = flce.flce_set_schedule(schedule)
    try:
        sizes = [flce.flce_workspace_size(p, op) for op in (0, 1, 2)]
    finally:
        flce.flce_set_schedule(prev)
    assert all(s > 0 for s in sizes)
    logits_bytes = w.BT * w.V * (2 if w.dtype == "bf16" else 4)
    if w.BT * w.V <= 1 << 20:
        return
    if schedule == 1 or w.dtype != "bf16":
        assert sizes[2] >= max(sizes[0], sizes[1])
        assert sizes[2] < logits_bytes
    else:
        per_row = 8 * -(-w.V // 256) + 16  # LSE partials, lse, target, NLL
        dx_slabs = 16 * w.BT * w.H  # at most eight fp32 K-split slabs of half the rows
        assert sizes[2] <= (0.5 * logits_bytes + 4 * w.V * w.H + per_row * w.BT + dx_slabs
                            + 4096)


def test_gpt2_workspace_below_the_pages_softmax_tensor():
    """PR #126348 sizes the llm.c softmax tensor at ~3 GB; the fused op's whole
    scratch space must stay well below one such tensor."""
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "pages_values.json")))
    t = g["llmc_softmax_tensor"]
    p = flce.make_problem(t["batch_size"] * t["sequence_length"], 768, t["vocab_size"])
    assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) < 0.5 * t["approx_bytes"]


def test_workspace_zero_for_invalid_problems():
    bad = [flce.make_problem(-1, 64, 10), flce.make_problem(4, 0, 10),
           flce.make_problem(4, 64, 0), flce.make_problem(4, 12, 10),
           flce.make_problem(4, 64, 10, dtype=7), flce.make_problem(4, 64, 1 << 31)]
    for p in bad:
        assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) == 0
    assert flce.flce_workspace_size(flce.make_problem(4, 64, 10), 9) == 0


class _Fake:
    """Stand-in for a device tensor: an address and a size (never dereferenced)."""

    def __init__(self, addr, nbytes=1 << 40):
        self.addr, self.nbytes = addr, nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


A = 1 << 20  # a 256-byte aligned fake address


def _fwd(p, X=A, W=A, lab=A, loss=A, lse=A, ws=A, ws_bytes=1 << 40):
    return binding.lib().flce_forward(p, X, W, lab, loss, lse, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(X=A + 8), 3), (dict(W=A + 2), 3), (dict(lab=A + 4), 3), (dict(ws=A + 128), 3),
    (dict(loss=A + 2), 3), (dict(W=0), 1), (dict(X=0), 1), (dict(loss=0), 1), (dict(ws=0), 1),
    (dict(ws_bytes=100), 4)])
def test_forward_host_checks(kw, status):
    import ctypes
    p = flce.make_problem(64, 64, 512)
    assert _fwd(ctypes.byref(p), **kw) == status


def test_problem_checks_before_any_launch():
    import ctypes
    L = binding.lib()
    assert L.flce_forward(None, A, A, A, A, A, A, 1 << 40, None) == 1
    for p, st in [(flce.make_problem(64, 12, 512), 3), (flce.make_problem(64, 64, 512, dtype=3), 2),
                  (flce.make_problem(-5, 64, 512), 1),
                  # 2^20 x 2^24 logits: more 128 x 256 tiles than 32-bit tile ids allow
                  (flce.make_problem(1 << 20, 64, 1 << 24), 2),
                  # fp32 CUDA-core kernels: at most 65535 blocks of 32 rows
                  (flce.make_problem(65535 * 32 + 1, 64, 512, dtype=flce.FLCE_FP32), 2)]:
        assert L.flce_fused(ctypes.byref(p), A, A, A, 1.0, A, A, A, A, 1 << 40, None) == st
        assert L.flce_backward(ctypes.byref(p), A, A, A, A, A, A, A, A, 1 << 40, None) == st
    p = flce.make_problem(64, 64, 512)
    p.dw_fp32 = 2
    assert L.flce_forward(ctypes.byref(p), A, A, A, A, A, A, 1 << 40, None) == 1
    # in-op label shift: T must divide BT and be >= 0
    for T in (-1, 48):
        p = flce.make_problem(64, 64, 512, shift_seq_len=T)
        assert L.flce_forward(ctypes.byref(p), A, A, A, A, A, A, 1 << 40, None) == 1
        assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) == 0
    p = flce.make_problem(64, 64, 512, shift_seq_len=32)
    base = flce.flce_workspace_size(flce.make_problem(64, 64, 512), flce.FLCE_OP_FUSED)
    assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) == base + 512  # 64 int64 labels
    p = flce.make_problem(64, 64, 512)
    assert L.flce_backward(ctypes.byref(p), A, A, A, A, 0, A, A, A, 1 << 40, None) == 1
    assert L.flce_backward(ctypes.byref(p), A, A, A, A, A, A + 8, A, A, 1 << 40, None) == 3
    assert L.flce_fused(ctypes.byref(p), A, A, A, 1.0, A, A, A, A, 10, None) == 4
    assert L.flce_get_device_status(None, None, None, None) == 1


def test_binding_raises_with_status():
    p = flce.make_problem(64, 64, 512)
    ws = _Fake(A + 1)
    with pytest.raises(flce.FlceError) as e:
        binding.flce_forward(p, _Fake(A), _Fake(A), _Fake(A), _Fake(A), _Fake(A), ws, stream=0)
    assert e.value.status == 3


def test_kernel_code_hash_ignores_comments_only(tmp_path):
    """bench.py keys its recorded DRAM traffic to csrc_sha16(): editing a
    comment keeps the hash, editing code changes it."""
    import shutil
    import bench
    src = os.path.join(ROOT, "linear_cross_entropy_tiles_b200", "csrc")
    dst = tmp_path / "linear_cross_entropy_tiles_b200" / "csrc"
    shutil.copytree(src, dst)
    base = bench.csrc_sha16(str(tmp_path))
    assert base == bench.csrc_sha16()
    f = dst / "aux_kernels.cuh"
    text = f.read_text()
    f.write_text(text + "\n// a new comment line\n/* and a block\n   comment */\n")
    assert bench.csrc_sha16(str(tmp_path)) == base
    f.write_text(text.replace("kStatusBadLabel = 5", "kStatusBadLabel = 6"))
    assert bench.csrc_sha16(str(tmp_path)) != base


def test_row_stride_checks_before_any_launch():
    """ldx/ldw/lddx/lddw: 0 means H; below H is invalid; a row pitch that is
    not a whole number of 16-byte units is misaligned; both found on the
    host."""
    import ctypes
    L = binding.lib()
    ok = flce.make_problem(64, 64, 512, ldx=72, ldw=128, lddx=64, lddw=96)
    assert flce.flce_workspace_size(ok, flce.FLCE_OP_FUSED) > 0
    # strides do not change the workspace
    assert (flce.flce_workspace_size(ok, flce.FLCE_OP_FUSED)
            == flce.flce_workspace_size(flce.make_problem(64, 64, 512), flce.FLCE_OP_FUSED))
    for field in ("ldx", "ldw", "lddx", "lddw"):
        for value, st in [(56, 1), (-8, 1), (68, 3), (1 << 31, 2)]:
            p = flce.make_problem(64, 64, 512, **{field: value})
            assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) == 0
            assert L.flce_fused(ctypes.byref(p), A, A, A, 1.0, A, A, A, A, 1 << 40, None) == st
    # fp32 rows: a stride of 68 elements is 272 bytes, a whole number of 16-byte units
    p = flce.make_problem(64, 64, 512, dtype=flce.FLCE_FP32, ldx=68)
    assert flce.flce_workspace_size(p, flce.FLCE_OP_FUSED) > 0


def test_ce_host_checks():
    import ctypes
    L = binding.lib()
    mk = flce.make_ce_problem
    p = mk(1000, 50257)
    fwd = flce.flce_ce_workspace_size(p, flce.FLCE_OP_FORWARD)
    bwd = flce.flce_ce_workspace_size(p, flce.FLCE_OP_BACKWARD)
    assert fwd >= 256 + 4 * 1000 and bwd == 256
    assert flce.flce_ce_workspace_size(p, flce.FLCE_OP_FUSED) == fwd   # flce_ce_fused
    assert flce.flce_ce_workspace_size(p, 9) == 0
    sh = mk(1000, 50257, shift_seq_len=100)
    assert flce.flce_ce_workspace_size(sh, flce.FLCE_OP_BACKWARD) == 256 + 8192  # 256-aligned
    for bad, st in [(mk(-1, 10), 1), (mk(4, 0), 1), (mk(4, 10, ld=9), 1), (mk(4, 10, ld_grad=3), 1),
                    (mk(4, 10, dtype=5), 2), (mk(4, 1 << 31), 2), (mk(6, 10, shift_seq_len=4), 1)]:
        assert flce.flce_ce_workspace_size(bad, flce.FLCE_OP_FORWARD) == 0
        assert L.flce_ce_forward(ctypes.byref(bad), A, A, A, A, A, 1 << 40, None) == st
        assert L.flce_ce_backward(ctypes.byref(bad), A, A, A, A, A, A, 1 << 40, None) == st
    ok = mk(4, 10)
    # bf16 logits need 2-byte alignment only (rows of odd V are fine), fp32 4
    assert L.flce_ce_forward(ctypes.byref(ok), A + 1, A, A, A, A, 1 << 40, None) == 3
    assert L.flce_ce_forward(ctypes.byref(mk(4, 10, dtype=flce.FLCE_FP32)), A + 2, A, A, A, A,
                             1 << 40, None) == 3
    assert L.flce_ce_forward(ctypes.byref(ok), A, A + 4, A, A, A, 1 << 40, None) == 3
    assert L.flce_ce_forward(ctypes.byref(ok), A, A, A, A, A + 8, 1 << 40, None) == 3
    assert L.flce_ce_forward(ctypes.byref(ok), A, A, A, A, A, 10, None) == 4
    assert L.flce_ce_forward(ctypes.byref(ok), A, A, 0, A, A, 1 << 40, None) == 1
    assert L.flce_ce_backward(ctypes.byref(ok), A, A, A, 0, A, A, 1 << 40, None) == 1
    assert L.flce_ce_backward(ctypes.byref(ok), A, A, A, A, A + 1, A, 1 << 40, None) == 3
    # flce_ce_fused: loss required, lse optional, dlogits aligned to the element
    assert L.flce_ce_fused(ctypes.byref(ok), A, A, 1.0, 0, A, A, A, 1 << 40, None) == 1
    assert L.flce_ce_fused(ctypes.byref(ok), A, A, 1.0, A, A, A + 1, A, 1 << 40, None) == 3
    assert L.flce_ce_fused(ctypes.byref(ok), A, A, 1.0, A, A, A, A, 10, None) == 4
    for bad, st in [(mk(4, 10, ld=9), 1), (mk(4, 10, dtype=5), 2)]:
        assert L.flce_ce_fused(ctypes.byref(bad), A, A, 1.0, A, A, A, A, 1 << 40, None) == st


def test_binding_checks_tensors_against_the_problem():
    """The binding raises before taking a pointer when a tensor's layout,
    dtype or device differs from what the problem says (no GPU needed:
    every case fails a check first)."""
    import torch
    X = torch.zeros(8, 64, dtype=torch.bfloat16)
    W = torch.zeros(40, 64, dtype=torch.bfloat16)
    lab = torch.zeros(8, dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA"):
        flce.fused(X, W, lab)                       # host tensors never reach a kernel
    with pytest.raises(ValueError, match="unit-stride"):
        binding._problem_of(torch.zeros(64, 8, dtype=torch.bfloat16).t(), W, -100, 0.0)
    with pytest.raises(ValueError, match="both"):
        binding._problem_of(X, W.float(), -100, 0.0)
    wide = torch.zeros(8, 96, dtype=torch.bfloat16)
    p = binding._problem_of(wide[:, 16:80], W, -100, 0.0)
    assert (p.ldx, p.ldw, p.H) == (96, 64, 64)      # a column slice: row stride 96
    p = flce.make_problem(8, 64, 40)
    for kw, msg in [(dict(X=X[:, :32]), "shape"), (dict(labels=lab.int()), "int64"),
                    (dict(X=wide[:, :64]), "row stride 96, the problem says 64"),
                    (dict(X=X), "CUDA")]:
        with pytest.raises(ValueError, match=msg):
            binding._check_flce(p, **kw)
    with pytest.raises(ValueError, match="CUDA"):
        flce.ce_forward(torch.zeros(4, 10), torch.zeros(4, dtype=torch.int64))


@pytest.mark.parametrize("name", ["gpt2_small", "llama3_8b", "gemma2_softcap"])
def test_workspace_below_one_logits_tensor_when_capped_or_fp32_dW(name):
    """The survey's bound on peak extra HBM, below one bf16 BT x V tensor,
    holds in two modes: under a workspace cap of exactly that size (the
    automatic schedule then gives up the fused-in-forward plan, or narrows
    the recompute chunk, as needed), and with an fp32 dW, where the
    fused-in-forward schedule keeps its running sum in dW itself."""
    w = inputs.WORKLOADS[name]
    logits_bytes = 2 * w.BT * w.V
    p = flce.make_problem(w.BT, w.H, w.V, flce.FLCE_BF16, softcap=w.softcap)
    free = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
    prev = flce.flce_set_workspace_limit(logits_bytes)
    try:
        capped = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
        # a forced schedule ignores the cap
        old = flce.flce_set_schedule(flce.FLCE_SCHEDULE_FUSED_FORWARD)
        forced = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
        flce.flce_set_schedule(old)
        # a cap below every plan: the smallest recompute plan
        flce.flce_set_workspace_limit(1)
        smallest = flce.flce_workspace_size(p, flce.FLCE_OP_FUSED)
    finally:
        flce.flce_set_workspace_limit(prev)
    assert capped < logits_bytes and (capped == free or capped < free)
    assert forced == free and 0 < smallest <= capped
    p32 = flce.make_problem(w.BT, w.H, w.V, flce.FLCE_BF16, softcap=w.softcap, dw_fp32=1)
    f32 = flce.flce_workspace_size(p32, flce.FLCE_OP_FUSED)
    assert f32 < logits_bytes
    assert free - f32 == -(-w.V * w.H * 4 // 256) * 256     # exactly the fp32 sum


def test_dw_fp32_problem_checks():
    import ctypes
    L = binding.lib()
    # fp32 dW rows: a stride of 68 floats is 272 bytes (16-byte multiple); as
    # bf16 it would be 136 bytes (not)
    assert flce.flce_workspace_size(flce.make_problem(64, 64, 512, lddw=68, dw_fp32=1), 2) > 0
    p = flce.make_problem(64, 64, 512, lddw=68)
    assert L.flce_fused(ctypes.byref(p), A, A, A, 1.0, A, A, A, A, 1 << 40, None) == 3
    for bad in (-1, 2):
        p = flce.make_problem(64, 64, 512, dw_fp32=bad)
        assert L.flce_fused(ctypes.byref(p), A, A, A, 1.0, A, A, A, A, 1 << 40, None) == 1


def test_vocab_parallel_host_checks():
    import ctypes
    L = binding.lib()
    p = flce.make_problem(64, 64, 300)
    for op in (0, 1):
        assert flce.binding.flce_vp_workspace_size(p, op) > 0
    assert flce.binding.flce_vp_workspace_size(p, 2) == 0
    sh = flce.make_problem(64, 64, 300, shift_seq_len=32)
    assert flce.binding.flce_vp_workspace_size(sh, 0) == 0
    for args, st in [((p, 0, 299), 1), ((p, -1, 1000), 1), ((p, 800, 1000), 1),
                     ((sh, 0, 1000), 2), ((p, 0, 1 << 31), 2)]:
        pr, off, tot = args
        assert L.flce_vp_forward(ctypes.byref(pr), off, tot, A, A, A, A, A, 1 << 40, None) == st
        assert L.flce_vp_backward(ctypes.byref(pr), off, tot, A, A, A, A, A, A, A, A, 1 << 40,
                                  None) == st
    assert L.flce_vp_forward(ctypes.byref(p), 0, 300, A, A, A, A + 2, A, 1 << 40, None) == 3
    assert L.flce_vp_forward(ctypes.byref(p), 0, 300, A, A, A, A, A, 10, None) == 4
    assert L.flce_vp_combine(ctypes.byref(p), 0, A, A, A, A, A, 1 << 40, None) == 1
    assert L.flce_vp_combine(ctypes.byref(p), 2, A, A, A, A, A, 100, None) == 4
    assert L.flce_vp_backward(ctypes.byref(p), 0, 300, A, A, A, A, A, A + 8, A, A, 1 << 40,
                              None) == 3


def test_sliced_call_host_checks():
    """flce_fused_global_sliced rejects a slice count outside [1, 64] and a
    NULL event before any CUDA call; flce_dw_slice_rows gives whole 256-row
    tiles that cover V."""
    import ctypes
    L = binding.lib()
    p = flce.make_problem(64, 64, 512)
    ev = (ctypes.c_void_p * 2)(A, A)
    args = (ctypes.byref(p), A, A, A, None, 1.0, A, A, A, A, 1 << 40)
    assert L.flce_fused_global_sliced(*args, 0, ev, None) == 1
    assert L.flce_fused_global_sliced(*args, 65, ev, None) == 1
    assert L.flce_fused_global_sliced(*args, 2, None, None) == 1
    assert L.flce_fused_global_sliced(*args, 2, (ctypes.c_void_p * 2)(A, None), None) == 1
    assert flce.flce_dw_slice_rows(128256, 8) == 16128
    assert flce.flce_dw_slice_rows(1000, 8) == 256
    assert flce.flce_dw_slice_rows(0, 4) == 0 and flce.flce_dw_slice_rows(10, 0) == 0
    assert flce.flce_dw_slice_rows(10, 65) == 0
    for V, n in ((128256, 8), (256000, 3), (50257, 64), (1, 1), (300, 2)):
        b = flce.dw_slice_bounds(V, n)
        assert len(b) == n and b[0][0] == 0 and b[-1][1] == V
        assert all(x1 == y0 for (_, x1), (y0, _) in zip(b, b[1:]))
        assert all((y - x) % 256 == 0 or y == V for x, y in b)


def test_recorded_traffic_and_profiles_describe_this_build():
    """bench.py's DRAM-traffic table and the ncu summaries under profiles/
    name the hash of the kernel sources they were captured from; both must
    describe the sources as they stand (a kernel change needs new captures)."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    h = bench.csrc_sha16()
    assert all(t["csrc_sha16"] == h for t in bench.TRAFFIC.values())
    prof = os.path.join(ROOT, "profiles")
    names = sorted(n for n in os.listdir(prof) if n.endswith(".md"))
    assert names
    for n in names:
        assert h in open(os.path.join(prof, n)).read(), n
