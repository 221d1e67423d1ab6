"""Benchmark: FLCE forward + backward (flce_fused) on the Llama-3-8B LM head.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one flce_fused call over one batch of synthetic inputs already
resident in HBM: labels check, then per row chunk the forward GEMM (logits,
per-row sum-exp, q = exp(y - R) stored in bf16 against one reference per
row), the per-row lse / scale / label-column pass, the dX GEMM (rows scaled
by their factor) and the accumulating dW GEMM, then the loss (the fused-in-forward schedule;
BT < 512 uses the two-pass recompute schedule).  Prints one JSON line.

Multi-GPU: one process per GPU (torchrun), data parallel over rows (weak
scaling: every rank holds BT rows of a global batch of N*BT rows and the same
W).  Each timed step counts the rank's non-ignored labels, all-reduces that
count (the divisor of the global mean), runs flce_fused_global (dW written
in fp32), and all-reduces the loss shares and the fp32 dW over NCCL.  --parallel replicas
runs independent copies instead (no collective).  Time is the max over ranks
of the device-timed region; value = tokens of all ranks / that time.

--workload ce_llmc times the cross-entropy path for callers that already
hold the logits (flce_ce_forward + flce_ce_backward) on PyTorch PR #126348's
llm.c tensor (32 x 1024 rows, V = 50257, bf16): HBM-bound, one read of the
logits forward, one read and one write backward.

The headline loop is timed with two CUDA events and nothing else; per-kernel
times (for the roofline and the shares) come from a second, shorter loop
with an event pair around every launch.

--impl reference times the fp64 CPU oracle (the only reference this build
has) on a bounded row sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("FLCE fwd+bwd tokens/s and TFLOP/s (% of B200 BF16 peak); peak extra HBM GB")

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel kind, from single-kernel ncu captures of the named workload (the
# commands and the per-launch figures are kept under profiles/).  They
# describe the kernel code whose hash (csrc_sha16) is recorded with them and
# are reported as null for any other build or workload.
TRAFFIC = {
    ("llama3_8b", "auto"): {
        "csrc_sha16": "8dea23cbe5ebac1f",
        "bytes_per_launch": {"lse_q_gemm": 2.3815e9, "dx_gemm": 5.5945e9, "dw_acc_gemm": 5.0345e9,
                             "lse_q": 0.0255e9}},
    ("gpt2_small", "auto"): {
        "csrc_sha16": "8dea23cbe5ebac1f",
        "bytes_per_launch": {"lse_q_gemm": 0.890e9, "dx_gemm": 1.0545e9,
                             "dw_acc_gemm": 1.183e9}},
    ("ce_llmc", "auto"): {
        "csrc_sha16": "8dea23cbe5ebac1f",
        "bytes_per_launch": {"ce_forward": 3.298e9, "ce_backward": 6.542e9,
                             "ce_fused": 6.531e9}},
}


def csrc_sha16(root=None):
    """Hash of the CUDA sources' code: comments and whitespace are stripped,
    so that editing a comment keeps the recorded DRAM traffic valid while
    any change to the code voids it."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    base = root or ROOT
    for f in sorted(glob.glob(os.path.join(base, "linear_cross_entropy_tiles_b200", "csrc", "*"))):
        with open(f, "r", encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(os.path.basename(f).encode())
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


L2_BYTES = 126 * 2 ** 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "flce_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world == 1 and args.parallel == "dp" and args.impl == "ours":
        # A one-rank group, so that the data-parallel step's collectives run.
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if "MASTER_PORT" not in os.environ:
            import socket
            s = socket.socket()
            s.bind(("127.0.0.1", 0))
            os.environ["MASTER_PORT"] = str(s.getsockname()[1])
            s.close()
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
    if world > 1 or (args.parallel == "dp" and args.impl == "ours"):
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def finish(world):
    barrier(world)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(w, X, W, labels, rows: int):
    """Time the fp64 oracle (as it stands) on `rows` rows of the workload."""
    import oracle
    from linear_cross_entropy_tiles_b200 import inputs
    R = inputs.sample_rows(w.BT, rows, seed=7)
    Xs = X[R].cpu()
    Wc = W.cpu()
    lab = labels[R].cpu()
    nv = int((labels != inputs.IGNORE_INDEX).sum().item())
    xa, tag = inputs.oracle_view(Xs)
    wa, _ = inputs.oracle_view(Wc)
    t0 = time.perf_counter()
    oracle.flce(xa, wa, lab.numpy(), softcap=w.softcap, n_valid=nv, dtype=tag)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": "%d of %d rows (full V=%d, H=%d), fp64 forward+backward incl. dW "
                      "contribution of those rows; %.2f s" % (rows, w.BT, w.V, w.H, dt)}


def run_reference(args, world, rank):
    """The oracle arm: fp64 CPU oracle on bounded row samples, rank 0 only."""
    if rank != 0:
        return
    from linear_cross_entropy_tiles_b200 import inputs
    if args.workload.startswith("ce_"):
        w = inputs.CE_WORKLOADS[args.workload]
        Z, labels = inputs.make_ce_workload(w, device="cuda")
        rows = args.ce_cpu_rows
        sample, metric, config = (lambda: ce_oracle_sample(w, Z, labels, rows), CE_METRIC,
                                  ce_config(w, world))
    else:
        w = inputs.WORKLOADS[args.workload]
        X, W, labels = inputs.make_workload(w, device="cuda")
        rows = args.cpu_rows
        sample, metric, config = (lambda: cpu_oracle_sample(w, X, W, labels, rows), METRIC,
                                  workload_config(w, world))
    times = []
    cb = None
    for i in range(args.warmup + args.steps):
        cb = sample()
        if i >= args.warmup:
            times.append(rows / cb["value"])
    t = sum(times) / len(times)
    value = rows / t
    line = {"impl": "reference", "metric": metric, "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config,
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def traffic_of(kind, workload, schedule, bt_override):
    """DRAM bytes per launch of `kind` from the recorded captures, or None when
    no capture describes this build, workload and schedule."""
    t = TRAFFIC.get((workload, schedule))
    if bt_override or t is None or csrc_sha16() != t["csrc_sha16"]:
        return None
    return t["bytes_per_launch"].get(kind)


def profile_kinds(step, n_steps, launches_per_step):
    """Run n_steps of `step` with an event pair around every library launch;
    return {kind: [total ms, launches]}."""
    import linear_cross_entropy_tiles_b200 as flce
    torch.cuda.synchronize()
    flce.flce_profile_start(launches_per_step * n_steps + 8)
    for _ in range(n_steps):
        step()
    torch.cuda.synchronize()
    by_kind = {}
    for name, t in flce.flce_profile_stop():
        k = by_kind.setdefault(name, [0.0, 0])
        k[0] += t
        k[1] += 1
    return by_kind


def cublas_floor(w, X, W, compute, stream, rounds):
    """The same shape's three dense GEMMs in cuBLAS (torch.mm): logits
    X W^T into a bf16 BT x V buffer, then G W and G^T X from it -- the
    6 BT H V FLOP of the fused call with no softmax, no exponentials and no
    per-row work -- timed in alternation with the fused call on the same
    stream (rounds of a few calls each), so both see the same clocks.  V is
    padded to a multiple of 64 for cuBLAS (rows of 16-byte multiples keep
    it on its tensor-core kernels).  Medians over the rounds, ms per call."""
    Vp = (w.V + 63) // 64 * 64
    Wp = torch.zeros(Vp, w.H, dtype=W.dtype, device=W.device)
    Wp[:w.V].copy_(W)
    G = torch.empty(w.BT, Vp, dtype=X.dtype, device=X.device)
    dXc, dWc = torch.empty_like(X), torch.empty_like(Wp)
    parts = {"forward": lambda: torch.mm(X, Wp.t(), out=G),
             "dx": lambda: torch.mm(G, Wp, out=dXc),
             "dw": lambda: torch.mm(G.t(), X, out=dWc)}

    def three():
        for f in parts.values():
            f()

    def timed(f, n):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            f()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / n

    n = 10 if w.BT * w.H * w.V < 8e12 else 6
    for f in (compute, three, compute, three):
        f()
    torch.cuda.synchronize()
    rows = []
    for _ in range(rounds):
        r = {"ours": timed(compute, n), "cublas": timed(three, n)}
        r.update({k: timed(f, n) for k, f in parts.items()})
        rows.append(r)
    med = {k: sorted(r[k] for r in rows)[len(rows) // 2] for k in rows[0]}
    del G, dXc, dWc, Wp
    torch.cuda.empty_cache()
    return {"ms": med["cublas"], "ours_ms_interleaved": med["ours"],
            "per_gemm_ms": {k: med[k] for k in parts}, "rounds": rounds, "calls_per_round": n,
            "v_padded": Vp, "api": "torch.mm (cuBLAS), bf16 in/out, fp32 accumulate"}


def time_steps(step, steps, world, stream, sampler=None):
    """Device time of `steps` calls of step() between two CUDA events on the
    launching stream, barriers and synchronisation on both sides; ms per
    step, max over ranks."""
    barrier(world)
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
        time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler is not None else None
    return max_over_ranks(t0.elapsed_time(t1) / steps, world), clocks


def workload_config(w, world, parallel="replicas"):
    return {"workload": "%s LM head: BT=%d H=%d V=%d %s%s, %.0f%% ignored"
                        % (w.name, w.BT, w.H, w.V, w.dtype,
                           (" softcap %g" % w.softcap) if w.softcap else "",
                           100 * w.ignore_frac),
            "BT": w.BT, "H": w.H, "V": w.V, "softcap": w.softcap,
            "ignore_frac": w.ignore_frac, "seed": w.seed,
            "l2": "inputs larger than L2 (W is %.2f GB vs 126 MB L2)" % (w.V * w.H * 2 / 1e9),
            "parallelism": "%s x%d" % (parallel, world), "schedule": SCHEDULE[0]}


SCHEDULE = ["auto"]


def run_ragged(args, world, rank):
    """Page 1's ragged-BT sweep: 82 flce_fused calls with BT drawn by the
    issue's formula (H=4096, V=128256, bf16, 5% ignored), each on its own
    seeded inputs; per-BT device time and aggregate tokens/s."""
    import linear_cross_entropy_tiles_b200 as flce
    from linear_cross_entropy_tiles_b200 import build, inputs
    build.build()
    flce.flce_set_schedule({"auto": 0, "recompute": 1, "fused_fwd": 2}[args.schedule])
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    bts = inputs.ragged_bt_list()
    if args.ragged_limit:
        bts = bts[:args.ragged_limit]
    per_bt = []
    total_ms = 0.0
    launches = 0
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    for i, BT in enumerate(bts):
        w = inputs.ragged_workload(i, BT)
        X, W, labels = inputs.make_workload(w, device=dev)
        p = flce.make_problem(w.BT, w.H, w.V, X.dtype)
        ws = flce.workspace(p, flce.FLCE_OP_FUSED, dev)
        loss = torch.empty(1, dtype=torch.float32, device=dev)
        dX, dW = torch.empty_like(X), torch.empty_like(W)
        flce.flce_fused(p, X, W, labels, 1.0, loss, dX, dW, ws, stream)  # warm-up
        launches_call = flce.flce_last_launch_count()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.ragged_reps):
            flce.flce_fused(p, X, W, labels, 1.0, loss, dX, dW, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1) / args.ragged_reps, world)
        status, _ = flce.flce_get_device_status(ws)
        if status != 0:
            raise SystemExit("device status %d at BT=%d" % (status, BT))
        total_ms += ms
        launches += launches_call * args.ragged_reps
        per_bt.append({"BT": BT, "ms": round(ms, 4), "tokens_per_s": round(world * BT / ms * 1e3),
                       "tflops": round(6.0 * BT * w.H * w.V / ms / 1e9, 1)})
        del X, W, labels, ws, dX, dW
    clocks = sampler.stop()
    peaks = load_peaks()
    tot_tokens = sum(b["BT"] for b in per_bt)
    value = world * tot_tokens / (total_ms / 1e3)
    tflops = 6.0 * tot_tokens * 4096 * 128256 / (total_ms / 1e3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.ragged_reps, "warmup": 1, "ms_per_step": total_ms / len(per_bt),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "ragged BT sweep: %d calls, BT %d..%d (sum %d), H=4096, "
                                   "V=128256, bf16, 5%% ignored" % (len(per_bt), min(bts),
                                                                    max(bts), tot_tokens),
                       "parallelism": "replicas x%d" % world, "schedule": args.schedule,
                       "l2": "inputs larger than L2 (W is 1.05 GB)"},
            "tflops": tflops, "frac_of_bf16_peak": tflops / world / peaks["bf16"],
            "gpu_launches": launches, "clocks": clocks, "per_bt": per_bt}), flush=True)


CE_METRIC = ("cross-entropy from held logits, fwd+bwd tokens/s and GB/s (% of B200 HBM "
             "copy bandwidth)")


def ce_config(w, world):
    return {"workload": "%s: logits BT=%d x V=%d %s (PyTorch PR #126348's llm.c tensor), "
                        "N(0, %.3f^2), %.0f%% ignored" % (w.name, w.BT, w.V, w.dtype, w.std,
                                                         100 * w.ignore_frac),
            "BT": w.BT, "V": w.V, "softcap": w.softcap, "seed": w.seed,
            "l2": "inputs larger than L2 (logits %.2f GB vs 126 MB L2)"
                  % (w.BT * w.V * 2 / 1e9),
            "parallelism": "replicas x%d" % world}


def ce_oracle_sample(w, Z, labels, rows):
    """Time the fp64 oracle's cross-entropy (forward and gradient) on `rows`
    rows of the logits."""
    import oracle
    from linear_cross_entropy_tiles_b200 import inputs
    R = inputs.sample_rows(w.BT, rows, seed=7)
    za, tag = inputs.oracle_view(Z[R].cpu())
    lab = labels[R].cpu().numpy()
    nv = int((labels != inputs.IGNORE_INDEX).sum().item())
    t0 = time.perf_counter()
    oracle.ce(za, lab, softcap=w.softcap, n_valid=nv, dtype=tag)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": "%d of %d rows (full V=%d), fp64 forward + logit gradient; %.2f s"
                      % (rows, w.BT, w.V, dt)}


def run_ce(args, world, rank):
    """flce_ce_forward + flce_ce_backward on logits resident in HBM."""
    import linear_cross_entropy_tiles_b200 as flce
    from linear_cross_entropy_tiles_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = inputs.CE_WORKLOADS[args.workload]
    if args.bt:
        import dataclasses
        w = dataclasses.replace(w, BT=args.bt)
    Z, labels = inputs.make_ce_workload(w, device=dev)
    stream = torch.cuda.current_stream()
    pf = flce.make_ce_problem(w.BT, w.V, Z.dtype, softcap=w.softcap)
    ws_f = flce.ce_workspace(pf, flce.FLCE_OP_FORWARD, dev)
    ws_b = flce.ce_workspace(pf, flce.FLCE_OP_BACKWARD, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    lse = torch.empty(w.BT, dtype=torch.float32, device=dev)
    dloss = torch.ones(1, dtype=torch.float32, device=dev)
    dZ = torch.empty_like(Z)

    fused = args.ce_mode == "fused"
    ws_u = flce.ce_workspace(pf, flce.FLCE_OP_FUSED, dev) if fused else None

    def step():
        if fused:  # one read and one write of the logits
            flce.flce_ce_fused(pf, Z, labels, 1.0, loss, lse, dZ, ws_u, stream)
            return
        flce.flce_ce_forward(pf, Z, labels, loss, lse, ws_f, stream)
        flce.flce_ce_backward(pf, Z, labels, lse, dloss, dZ, ws_b, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status, n_valid = flce.flce_get_device_status(ws_u if fused else ws_f)
    if status != 0:
        raise SystemExit("device status %d after warm-up" % status)
    if fused:
        step()
        launches_per_step = flce.flce_last_launch_count()
    else:
        flce.flce_ce_forward(pf, Z, labels, loss, lse, ws_f, stream)
        launches_per_step = flce.flce_last_launch_count()
        flce.flce_ce_backward(pf, Z, labels, lse, dloss, dZ, ws_b, stream)
        launches_per_step += flce.flce_last_launch_count()
    sampler = ClockSampler(torch.cuda.current_device())
    ms, clocks = time_steps(step, args.steps, world, stream, sampler)
    peaks = load_peaks()
    by_kind = profile_kinds(step, max(1, min(args.steps, args.prof_steps)), launches_per_step)
    total = sum(v[0] for v in by_kind.values())
    elem = w.BT * w.V * (2 if w.dtype == "bf16" else 4)
    # The backward moves two of the step's three logits-sized passes; the
    # fused call both of its two.
    bytes_per_launch = {"ce_forward": float(elem), "ce_backward": 2.0 * elem,
                        "ce_fused": 2.0 * elem}
    step_bytes = 2.0 * elem if fused else w.bytes_per_step
    dom = max(by_kind, key=lambda n: by_kind[n][0])
    dom_ms = by_kind[dom][0] / by_kind[dom][1]
    achieved = bytes_per_launch.get(dom, 0.0) / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "peak_kind": "%s HBM copy bandwidth" % peaks["source"],
                "bytes_per_launch": bytes_per_launch.get(dom), "avg_launch_ms": dom_ms,
                "traffic": traffic_of(dom, args.workload, "auto", args.bt),
                "per_kernel_gbs": {k: round(bytes_per_launch[k] / (v[0] / v[1] / 1e3) / 1e9, 1)
                                   for k, v in by_kind.items() if k in bytes_per_launch},
                "shares": {k: round(v[0] / total, 4) for k, v in sorted(by_kind.items())}}
    e2e = None
    if not args.no_e2e:
        # The step's data (the logits and labels) in from pinned host memory,
        # the loss out; the logit gradient stays on the device for the LM
        # head's backward (--e2e-copies all copies it out too).
        copy_all = args.e2e_copies == "all"
        Zh = Z.cpu().pin_memory()
        Lh = labels.cpu().pin_memory()
        lossh = torch.empty(1, dtype=torch.float32).pin_memory()
        dZh = torch.empty(Z.shape, dtype=Z.dtype).pin_memory() if copy_all else None

        def e2e_step():
            Z.copy_(Zh, non_blocking=True)
            labels.copy_(Lh, non_blocking=True)
            step()
            lossh.copy_(loss, non_blocking=True)
            if copy_all:
                dZh.copy_(dZ, non_blocking=True)

        e2e_step()
        ems, _ = time_steps(e2e_step, args.e2e_steps, world, stream)
        e2e = {"value": world * w.BT / (ems / 1e3), "unit": "tokens/s", "ms_per_step": ems,
               "h2d_bytes_per_step": Zh.numel() * Zh.element_size() + Lh.numel() * 8,
               "d2h_bytes_per_step": 4 + (dZh.numel() * dZh.element_size() if copy_all else 0),
               "copies": ("logits, labels in; loss, dlogits out" if copy_all else
                          "logits, labels in; loss out (dlogits stays on the device)"),
               "api": ("linear_cross_entropy_tiles_b200 flce_ce_fused (C ABI)" if fused else
                       "linear_cross_entropy_tiles_b200 flce_ce_forward + flce_ce_backward "
                       "(C ABI)")}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = ce_oracle_sample(w, Z, labels, args.ce_cpu_rows)
    if rank == 0:
        print(json.dumps({
            "metric": CE_METRIC, "value": world * w.BT / (ms / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic", "config": ce_config(w, world),
            "gbs": step_bytes / (ms / 1e3) / 1e9,
            "frac_of_hbm": step_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "bytes_per_step": step_bytes, "ce_mode": args.ce_mode, "n_valid": n_valid,
            "loss": float(loss.item()), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clocks}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama3_8b")
    ap.add_argument("--bt", type=int, default=0,
                    help="override BT of the workload (small cases for profiling)")
    ap.add_argument("--v", type=int, default=0,
                    help="override V of an LM-head workload (small cases for profiling "
                         "that keep the full-size K of every GEMM)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--schedule", default="auto", choices=["auto", "recompute", "fused_fwd"],
                    help="flce_fused schedule (auto: fused-in-forward for BT >= 512)")
    ap.add_argument("--cpu-rows", type=int, default=8)
    ap.add_argument("--ce-cpu-rows", type=int, default=8192)
    ap.add_argument("--ce-mode", default="separate", choices=["separate", "fused"],
                    help="ce_* workloads: flce_ce_forward + flce_ce_backward (the PR's two "
                         "passes), or flce_ce_fused (one read of the logits)")
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="timed end-to-end steps (0: as many as --steps)")
    ap.add_argument("--e2e-copies", default="data", choices=["data", "all"],
                    help="e2e host copies per step: the step's data in and the loss out "
                         "(default), or also W in and the gradients out")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cublas-floor", action="store_true",
                    help="also time the shape's three bare GEMMs in cuBLAS, alternating with "
                         "the fused call (adds \"cublas_3gemm\" to the line)")
    ap.add_argument("--floor-rounds", type=int, default=4)
    ap.add_argument("--ragged-reps", type=int, default=3)
    ap.add_argument("--ragged-limit", type=int, default=0)
    ap.add_argument("--prof-steps", type=int, default=20,
                    help="steps of the second, per-launch-timed loop")
    ap.add_argument("--dw-reduce", default="fp32", choices=["fp32", "bf16"],
                    help="data parallel: dtype in which dW is written and summed over ranks")
    ap.add_argument("--dw-slices", type=int, default=8,
                    help="data parallel: dW handed over in this many vocabulary slices, each "
                         "all-reduced on a side stream as soon as it is final (0: one "
                         "all-reduce after the call)")
    ap.add_argument("--parallel", default=None, choices=["dp", "replicas"],
                    help="with several ranks: data parallel over rows (default) or "
                         "independent replicas; 'dp' on one rank runs the same step "
                         "over a one-rank group")
    args = ap.parse_args()
    if args.e2e_steps <= 0:
        args.e2e_steps = args.steps
    world_env = int(os.environ.get("WORLD_SIZE", "1"))
    if args.parallel is None:
        args.parallel = "dp" if world_env > 1 else "replicas"
    if (args.workload == "ragged" or args.workload.startswith("ce_")) and args.parallel == "dp":
        # each ragged BT is a problem of its own; the CE path has no exchange
        args.parallel = "replicas"
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world, rank, local = dist_setup(args)
    SCHEDULE[0] = args.schedule
    if args.impl == "reference":
        run_reference(args, world, rank)
        finish(world)
        return

    if args.workload == "ragged":
        run_ragged(args, world, rank)
        finish(world)
        return

    if args.workload.startswith("ce_"):
        run_ce(args, world, rank)
        finish(world)
        return

    import linear_cross_entropy_tiles_b200 as flce
    from linear_cross_entropy_tiles_b200 import build, inputs
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    w = inputs.WORKLOADS[args.workload]
    if args.bt or args.v:
        import dataclasses
        w = dataclasses.replace(w, BT=args.bt or w.BT, V=args.v or w.V)
    if args.parallel == "dp" and world > 1:
        import dataclasses
        w = dataclasses.replace(w, seed=w.seed + 1000 * rank)  # each rank its own rows
    X, W, labels = inputs.make_workload(w, device=dev)
    if args.parallel == "dp" and world > 1:
        W = inputs.make_workload(dataclasses.replace(w, seed=inputs.WORKLOADS[args.workload].seed),
                                 device=dev, BT=1)[1]  # the same W on every rank
    flce.flce_set_schedule({"auto": 0, "recompute": 1, "fused_fwd": 2}[args.schedule])
    dp_mode = args.parallel == "dp"
    # Data parallel: each rank writes its dW share in fp32 and the ranks sum
    # it in fp32 (--dw-reduce bf16: bf16 shares summed in bf16).
    dw32 = dp_mode and args.dw_reduce == "fp32" and w.dtype == "bf16"
    p = flce.make_problem(w.BT, w.H, w.V, X.dtype, softcap=w.softcap, dw_fp32=int(dw32))
    torch.cuda.synchronize()
    ws = flce.workspace(p, flce.FLCE_OP_FUSED, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dX = torch.empty_like(X)
    dW = torch.empty(W.shape, dtype=torch.float32 if dw32 else W.dtype, device=dev)
    stream = torch.cuda.current_stream()

    n_valid_buf = torch.empty(1, dtype=torch.int64, device=dev)
    n_sl = args.dw_slices if dp_mode else 0
    slice_bounds = flce.dw_slice_bounds(w.V, n_sl) if n_sl > 0 else []
    slice_events = [torch.cuda.Event() for _ in slice_bounds]
    side = torch.cuda.Stream(device=dev) if n_sl > 0 else None

    def compute(X=X, labels=labels):
        if not dp_mode:
            flce.flce_fused(p, X, W, labels, 1.0, loss, dX, dW, ws, stream)
            return
        # Data-parallel step: the count of all ranks' non-ignored labels before
        # G is formed, then the loss shares and dW summed over the ranks --
        # slice by slice on a side stream as the slices become final, or in
        # one all-reduce after the call.
        flce.flce_count_valid(p, labels, n_valid_buf, stream)
        torch.distributed.all_reduce(n_valid_buf)
        if n_sl == 0:
            flce.flce_fused_global(p, X, W, labels, n_valid_buf, 1.0, loss, dX, dW, ws, stream)
            torch.distributed.all_reduce(loss)
            torch.distributed.all_reduce(dW)
            return
        flce.flce_fused_global_sliced(p, X, W, labels, n_valid_buf, 1.0, loss, dX, dW, ws,
                                      slice_events, stream)
        works = []
        with torch.cuda.stream(side):
            for ev, (a, b) in zip(slice_events, slice_bounds):
                side.wait_event(ev)
                if b > a:
                    works.append(torch.distributed.all_reduce(dW[a:b], async_op=True))
        torch.distributed.all_reduce(loss)
        for wk in works:
            wk.wait()

    def step():
        compute()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status, n_valid = flce.flce_get_device_status(ws)
    if status != 0:
        raise SystemExit("device status %d after warm-up" % status)
    # Our kernels per step: the fused call's, plus the label count in dp mode.
    launches_per_step = flce.flce_last_launch_count() + (1 if dp_mode else 0)
    extra_bytes = ws.numel()  # the only scratch memory; the library allocates nothing

    sampler = ClockSampler(torch.cuda.current_device())
    ms, clocks = time_steps(step, args.steps, world, stream, sampler)
    tokens_per_s = world * w.BT / (ms / 1e3)
    tflops = world * w.flops / (ms / 1e3) / 1e12
    peaks = load_peaks()

    # Per-kernel times from a second loop with events around every launch.
    prof_steps = max(1, min(args.steps, args.prof_steps))
    by_kind = profile_kinds(step, prof_steps, launches_per_step)
    total_prof = sum(v[0] for v in by_kind.values())
    dom = max(by_kind, key=lambda n: by_kind[n][0])
    # Algorithmic FLOPs per step of each GEMM kind: 2*BT*H*V each (the LSE and
    # G GEMMs recompute the logits X W^T, the dX / dW GEMMs are G W and G^T X).
    gemm_flops = 2.0 * w.BT * w.H * w.V
    flops_per_step = {k: gemm_flops for k in ("lse_gemm", "grad_gemm", "dx_gemm", "dw_gemm",
                                              "lse_q_gemm", "dw_acc_gemm", "simt_lse",
                                              "simt_grad", "simt_dx", "simt_dw")}
    dom_time_per_step = by_kind[dom][0] / prof_steps
    launches_dom = by_kind[dom][1] / prof_steps
    achieved = flops_per_step.get(dom, 0.0) / (dom_time_per_step / 1e3) / 1e12
    if w.dtype == "bf16":
        # A kernel of a few ms timed inside a sub-second region: the burst peak.
        bound, peak = "tensor", peaks["bf16"]
        peak_kind = ("%s burst dense bf16 (cuBLAS GEMM timed alone); frac_sustained divides "
                     "by the %s sustained figure (cuBLAS loop under the power cap)"
                     % (peaks["source"], peaks["source"]))
    else:
        # fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
        bound, peak = "alu", 148 * 128 * 2 * 1.965e9 / 1e12
        peak_kind = "fp32 CUDA-core FMA peak from unit counts and the max SM clock"
    roofline = {"bound": bound, "kernel": dom, "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "frac_sustained": (achieved / peaks["bf16_sustained"]
                                   if w.dtype == "bf16" else None),
                "peak_kind": peak_kind, "profiled_steps": prof_steps,
                "flops_per_launch": flops_per_step.get(dom, 0.0) / launches_dom,
                "avg_launch_ms": dom_time_per_step / launches_dom,
                "traffic": traffic_of(dom, args.workload, args.schedule, args.bt or args.v),
                "shares": {k: round(v[0] / total_prof, 4) for k, v in sorted(by_kind.items())}}

    # End to end through the public API with host buffers.  Per step, the
    # step's data -- the hidden states X and the labels -- come in from
    # pinned host memory and the loss goes back to the host (a training loop
    # logs it); W is a parameter resident on the device, and dX, dW are
    # consumed there by the rest of the backward pass and the optimizer.
    # --e2e-copies all also copies W in and dX, dW out every step.
    e2e = None
    if not args.no_e2e:
        copy_all = args.e2e_copies == "all"
        Xh = X.cpu().pin_memory()
        Wh = W.cpu().pin_memory() if copy_all else None
        Lh = labels.cpu().pin_memory()
        lossh = torch.empty_like(loss, device="cpu").pin_memory()
        dXh = torch.empty_like(dX, device="cpu").pin_memory() if copy_all else None
        dWh = torch.empty_like(dW, device="cpu").pin_memory() if copy_all else None

        # The step's data arrive as a training loop's loader delivers them:
        # step i's X and labels are copied into one of two device buffers on
        # a copy stream while step i - 1 computes (the first copy inside the
        # timed region too).  With --e2e-copies all every copy stays on the
        # compute stream, in order.
        bufs = [(X, labels), (torch.empty_like(X), torch.empty_like(labels))]
        cstream = torch.cuda.Stream(device=dev)
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        free = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(i):
            xb, lb = bufs[i % 2]
            cstream.wait_event(free[i % 2])  # step i - 2 is done with this buffer
            with torch.cuda.stream(cstream):
                xb.copy_(Xh, non_blocking=True)
                lb.copy_(Lh, non_blocking=True)
                ready[i % 2].record(cstream)

        def e2e_steps(n):
            if copy_all:
                for _ in range(n):
                    X.copy_(Xh, non_blocking=True)
                    W.copy_(Wh, non_blocking=True)
                    labels.copy_(Lh, non_blocking=True)
                    compute()
                    lossh.copy_(loss, non_blocking=True)
                    dXh.copy_(dX, non_blocking=True)
                    dWh.copy_(dW, non_blocking=True)
                return
            cstream.wait_stream(stream)  # the first copy starts inside the timed region
            issue_copy(0)
            for i in range(n):
                if i + 1 < n:
                    issue_copy(i + 1)
                stream.wait_event(ready[i % 2])
                compute(*bufs[i % 2])
                free[i % 2].record(stream)
                lossh.copy_(loss, non_blocking=True)

        e2e_steps(2)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_steps(args.e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world)
        h2d = Xh.numel() * Xh.element_size() + Lh.numel() * 8
        d2h = lossh.numel() * 4
        if copy_all:
            h2d += Wh.numel() * Wh.element_size()
            d2h += dXh.numel() * dXh.element_size() + dWh.numel() * dWh.element_size()
        e2e = {"value": world * w.BT / (ems / 1e3), "unit": "tokens/s", "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "copies": ("X, labels, W in; loss, dX, dW out, in order on the compute stream"
                          if copy_all else
                          "X, labels in (on a copy stream, one step ahead, two device "
                          "buffers); loss out (W resident, dX and dW stay on the device)"),
               "api": ("linear_cross_entropy_tiles_b200 flce_count_valid + flce_fused_global "
                       "(C ABI) + torch.distributed all-reduces" if dp_mode else
                       "linear_cross_entropy_tiles_b200.flce_fused (C ABI)")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w, X, W, labels, args.cpu_rows)
    floor = (cublas_floor(w, X, W, compute, stream, args.floor_rounds)
             if args.cublas_floor and world == 1 and w.dtype == "bf16" and not dp_mode else None)

    if rank == 0:
        line = {"metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
                "config": dict(workload_config(w, world, args.parallel),
                               **({"dw_reduce": "%s all-reduce in %s" % (
                                   "%d overlapped vocabulary slices" % n_sl if n_sl else
                                   "one call", "fp32" if dw32 else w.dtype)}
                                  if dp_mode else {})),
                "tflops": tflops, "frac_of_bf16_peak": tflops / world / peaks["bf16"],
                "frac_of_bf16_sustained": tflops / world / peaks["bf16_sustained"],
                "peak_basis": "%s: %.1f burst / %.1f sustained TFLOP/s dense bf16"
                              % (peaks["source"], peaks["bf16"], peaks["bf16_sustained"]),
                "peak_extra_hbm_gb": extra_bytes / 1e9,
                "n_valid": n_valid, "loss": float(loss.item()),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clocks}
        if floor is not None:
            line["cublas_3gemm"] = floor
        print(json.dumps(line), flush=True)
    finish(world)


if __name__ == "__main__":
    main()
