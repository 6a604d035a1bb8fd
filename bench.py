#!/usr/bin/env python
"""Benchmark of the mHC forward hot path (pre + post) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...        (one process per GPU)

One step = mhc_pre + mhc_post over one batch of T tokens (the whole hot path; F_out is a
given input, the sub-layer F itself is not part of the path).  Default workload: T = 16384
tokens (4 x 4096), n = 4 streams, d = 4096, bf16 storage, fp32 arithmetic, 1 % outlier
channels; inputs are synthetic and seeded (mhc_hyper_connections_b200.workloads).  A step's
buffers at that size (X 512 MiB + F_out 128 MiB + outputs) are far larger than L2, so no
flush is needed between steps; for a workload whose buffers are smaller than twice the L2,
the timed loop rotates through enough copies of them to cover three times the L2.

Multi-GPU: tokens are independent, so every rank runs its own T-token batch (weak
scaling, no data-path collective); the time is the max over ranks.

Prints ONE JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle instead, on
the host cores, over a bounded token sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "mHC pre+post tokens/s and achieved HBM GB/s (% of roofline), n=4 d=4096 bf16"
NOMINAL_HBM_GBS = 8000.0          # the target's roofline denominator ("~8 TB/s")
FALLBACK_HBM_GBS = 6650.0         # used only if MEASURED_PEAKS.json is absent

# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum) for
# the named kernel on the headline workload, with the sha256 of the kernel source it was
# measured on; reported as null once that source changes.
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum per launch, captured at half the token count
    # (X still twice the L2) and scaled x2 (profiles/ holds the commands and the raw counts)
    ("pre", "bf16_T16384_n4_d4096_outliers"): (int((270.448128 + 41.708544) * 2e6), "b2019263f3ba751a"),
    ("post", "bf16_T16384_n4_d4096_outliers"): (int((336.344832 + 210.074368) * 2e6), "e2d0eca830bf798b"),
    # the three launches of the two-pass path at T=4096: the projection and read-map kernels
    # scaled x2, the phi packing (no token dependence) once
    ("pre", "bf16_T8192_n8_d4096"): (int(((279.610624 + 0.082176 + 268.969216 + 5.862144) * 2 + 10.491904) * 1e6),
                                     "0811af1e75883c76"),
    # the six launches of one mhc_backward call at T=8192, scaled x2 (backward.cu + backward_tc.cu)
    ("backward", "bf16_T16384_n4_d4096_outliers"): (int((1286.790400 + 261.519104) * 2e6), "bab5f002ab08645e"),
}


def _hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


def _src_sha(rel):
    """sha256 prefix of a source file, or of several (a list) read one after another."""
    h = hashlib.sha256()
    try:
        for r in ([rel] if isinstance(rel, str) else rel):
            with open(os.path.join(ROOT, r), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return h.hexdigest()[:16]


def bytes_per_token(n, d, es):
    """Algorithmic HBM bytes per token.  pre: reads X (n d), writes x_in (d) and H (m fp32);
    post: reads X (n d), F_out (d), H_res + H_post ((n^2 + n) fp32), writes X' (n d)."""
    m = n * n + 2 * n
    pre = (n + 1) * d * es + 4 * m
    post = (2 * n + 1) * d * es + 4 * (n * n + n)
    return pre, post


L2_BYTES = 126 * 2 ** 20           # B200 L2 (the device's own figure is used when known)


def buffer_sets(T, n, d, es, l2_bytes=L2_BYTES):
    """How many copies of the step's buffers (X, F_out, x_in, H, X') the timed loop rotates
    through so that no step finds the previous step's data in L2: one when a single set is
    at least twice the L2, else enough sets to cover three times the L2 (at least four, at
    most 64: a step that small is bound by its launches, not by memory)."""
    m = n * n + 2 * n
    one = T * (2 * n + 2) * d * es + T * m * 4
    if one >= 2 * l2_bytes:
        return 1, one
    return min(64, max(4, -(-3 * l2_bytes // one))), one


def workload_config(w, world, l2_bytes=L2_BYTES):
    """The `config` object of the JSON line, the same for both arms: what the workload is,
    not how an arm ran it."""
    es = 2 if w.dtype == "bf16" else 4
    sets, one = buffer_sets(w.T, w.n, w.d, es, l2_bytes)
    mib = lambda b: f"{b / 2 ** 20:.0f} MiB" if b >= 2 ** 20 else f"{b / 2 ** 10:.0f} KiB"
    if sets == 1:
        l2 = (f"inputs larger than L2 (X {mib(w.T * w.n * w.d * es)} + F_out {mib(w.T * w.d * es)}; "
              f"one step's buffers {mib(one)} vs L2 {mib(l2_bytes)}), no flush")
    else:
        l2 = (f"{sets} buffer sets of {mib(one)} rotated between steps ({mib(sets * one)} vs L2 "
              f"{mib(l2_bytes)}), no flush")
    s = w.scalars()
    return {"workload": w.name.split("[")[0], "T": w.T, "n": w.n, "d": w.d, "storage": w.dtype,
            "tokens_per_gpu": w.T, "parallelism": f"replicas x{world} (token shards, no collective)",
            "l2": l2, "alpha": s["alpha_pre"], "t_max": s["t_max"], "eps": s["eps"]}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons, n_all = [], None, set(), 0
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            n_all += 1
            if not (t0 - 0.05 <= ts <= t1 + 0.15):
                continue
            try:
                sm.append(float(parts[2]))
                mx = float(parts[3])
            except ValueError:
                continue
            for nm, v in zip(names, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                    "samples": 0, "note": "no nvidia-smi sample fell inside the timed region"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm (oracle)
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from mhc_hyper_connections_b200 import workloads as wl

    w = wl.make_config(args.config)
    if args.tokens:
        w = w.tokens(np.arange(min(args.tokens, w.T)))
    cores = os.cpu_count() or 1
    used = oracle.threads_used(cores)
    s = w.scalars()

    def step(sub):
        X = sub.values(sub.X)
        F = sub.values(sub.F_out)
        t0 = time.perf_counter()
        _, H = oracle.mhc_pre(X, sub.phi, sub.b_pre, sub.b_post, sub.b_res, s["alpha_pre"],
                              s["alpha_post"], s["alpha_res"], eps=s["eps"], t_max=s["t_max"],
                              nthreads=cores)
        oracle.mhc_post(X, F, H, nthreads=cores)
        return time.perf_counter() - t0

    # size the per-step sample so the whole run stays within ~2 minutes
    cal = max(step(w.tokens(np.arange(min(64, w.T)))) / min(64, w.T), 1e-7)
    budget = 120.0 / max(1, args.steps + args.warmup)
    per_step = int(max(1, min(w.T, budget / cal)))
    rng = np.random.default_rng(0)
    subs = [w.tokens(np.sort(rng.choice(w.T, per_step, replace=False))) for _ in range(4)]
    for k in range(args.warmup):
        step(subs[k % 4])
    tot = 0.0
    for k in range(args.steps):
        tot += step(subs[k % 4])
    value = per_step * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": f"{per_step} random tokens of the {w.T}-token batch per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(w, seconds=10.0, chunk=1024, max_passes=64, single_seconds=3.0):
    """The oracle as it stands, on the host cores, over a bounded token sample: passes over
    the batch in chunks of `chunk` tokens (fp64 conversion outside the timed calls) until
    about `seconds` of timed oracle work has accumulated on all cores, then about
    `single_seconds` more on one thread."""
    import numpy as np

    import oracle
    cores = os.cpu_count() or 1
    used = oracle.threads_used(cores)
    s = w.scalars()

    def timed(nthreads, budget):
        done, t_sum, passes = 0, 0.0, 0
        while t_sum < budget and passes < max_passes:
            for c0 in range(0, w.T, chunk):
                sub = w.tokens(np.arange(c0, min(w.T, c0 + chunk)))
                X = sub.values(sub.X)
                F = sub.values(sub.F_out)
                t0 = time.perf_counter()
                _, H = oracle.mhc_pre(X, sub.phi, sub.b_pre, sub.b_post, sub.b_res, s["alpha_pre"],
                                      s["alpha_post"], s["alpha_res"], eps=s["eps"], t_max=s["t_max"],
                                      nthreads=nthreads)
                oracle.mhc_post(X, F, H, nthreads=nthreads)
                t_sum += time.perf_counter() - t0
                done += sub.T
                if t_sum >= budget:
                    break
            passes += 1
        return done, t_sum, passes

    done, t_sum, passes = timed(cores, seconds)
    one_done, one_t, _ = timed(1, single_seconds)
    return {"value": done / t_sum, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{done} tokens ({passes} pass(es) over the {w.T}-token batch in "
                      f"{chunk}-token chunks), {t_sum:.1f} s of fp64 oracle time on {used} "
                      f"OpenMP threads",
            "single_thread": {"value": one_done / one_t, "unit": "tokens/s", "cores": 1,
                              "sample": f"{one_done} tokens in {chunk}-token chunks from the "
                                        f"start of the batch, {one_t:.1f} s on one thread"}}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import mhc_hyper_connections_b200 as mhc
    from mhc_hyper_connections_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    from mhc_hyper_connections_b200 import dist as mdist

    def max_over_ranks(x):
        return mdist.max_over_ranks(x, device=dev)

    w = wl.make_config(args.config)
    if args.tokens:
        w = w.tokens(np.arange(min(args.tokens, w.T)))
    T, n, d = w.T, w.n, w.d
    es = 2 if w.dtype == "bf16" else 4
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    l2_bytes = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or L2_BYTES
    nsets, _ = buffer_sets(T, n, d, es, l2_bytes)
    X0, F0 = to_dev(w.X), to_dev(w.F_out)
    phi, b_pre, b_post, b_res = (to_dev(a) for a in (w.phi, w.b_pre, w.b_post, w.b_res))
    # nsets copies of the step's buffers, rotated so that no step reads the previous step's
    # data out of L2 (one set when a set is at least twice the L2)
    bufs = []
    for i in range(nsets):
        Xi, Fi = (X0, F0) if i == 0 else (X0.clone(), F0.clone())
        bufs.append(dict(X=Xi, F=Fi, x_in=torch.empty(T, d, dtype=tdt, device=dev),
                         H=torch.empty(T, w.m, dtype=torch.float32, device=dev),
                         Y=torch.empty_like(Xi)))
    X, F, x_in, H, Y = (bufs[0][k] for k in ("X", "F", "x_in", "H", "Y"))
    s = w.scalars()
    req = {"auto": mhc.PRE_AUTO, "generic": mhc.PRE_GENERIC, "cluster_tc": mhc.PRE_CLUSTER_TC,
           "two_pass_tc": mhc.PRE_TWO_PASS_TC}[args.pre_path]
    path = mhc.mhc_pre_path_for(T, n, d, tdt) if req == mhc.PRE_AUTO else req

    def pre(k=0):
        b = bufs[k % nsets]
        mhc.mhc_pre_with_path(b["X"], phi, b_pre, b_post, b_res, s["alpha_pre"], s["alpha_post"],
                              s["alpha_res"], s["eps"], s["t_max"], b["x_in"], b["H"], path=req)

    def post(k=0):
        b = bufs[k % nsets]
        mhc.mhc_post(b["X"], b["F"], b["H"], b["Y"])

    for k in range(args.warmup):
        pre(k)
        post(k)
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, events on the launching (current) stream
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank)
    clk.start()
    time.sleep(0.6)                       # let nvidia-smi start sampling
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record()
    for k in range(K):
        e = evs[k]
        e[0].record()
        pre(k)
        e[1].record()
        post(k)
        e[2].record()
    end.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier()
    time.sleep(0.3)
    clk.stop()
    ms_total = max_over_ranks(start.elapsed_time(end))
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    post_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    clocks = clk.summary(t_wall0, t_wall1)

    value = mdist.job_throughput(T, K, ms_total, world)
    peak, peak_src = _hbm_peak()
    by_pre, by_post = bytes_per_token(n, d, es)
    kern = {"pre": {"ms": pre_ms, "bytes_per_launch": by_pre * T,
                    "gbs": by_pre * T / (pre_ms / 1e3) / 1e9,
                    "path": {1: "generic", 2: "cluster_tc", 3: "two_pass_tc"}.get(path, str(path)),
                    "source": "mhc_hyper_connections_b200/csrc/" +
                              {2: "pre_tc.cu", 3: "pre_wide.cu"}.get(path, "pre_generic.cu")},
            "post": {"ms": post_ms, "bytes_per_launch": by_post * T,
                     "gbs": by_post * T / (post_ms / 1e3) / 1e9,
                     "source": "mhc_hyper_connections_b200/csrc/post.cu"}}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    traffic = None
    rec = NCU_TRAFFIC.get((dom, args.config))
    if rec and not args.tokens and rec[1] == _src_sha(kern[dom]["source"]):
        traffic = rec[0]                       # the capture is of the full token count
    achieved = kern[dom]["gbs"]
    roofline = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": kern[dom]["bytes_per_launch"]}
    b_dep = by_pre + by_post
    step_gbs = b_dep * T * world / (ms_total / 1e3 / K) / 1e9 / world
    hbm = {"B_dep_bytes_per_token": b_dep, "B_lit_bytes_per_token": (2 * n + 2) * d * es,
           "gbs_per_gpu": step_gbs, "frac_of_8TBs": step_gbs / NOMINAL_HBM_GBS,
           "frac_of_peak": step_gbs / peak, "peak_source": peak_src,
           "frac_of_8TBs_lit": (2 * n + 2) * d * es * T / (ms_total / 1e3 / K) / 1e9 / NOMINAL_HBM_GBS}

    # ---- end to end through the public API with host buffers (pinned), copies timed: one
    # mhc_forward_host call per step, which copies each chunk of tokens in, runs pre and post on
    # it and copies its outputs back, overlapping the two copy directions and the kernels
    e2e = None
    if not args.no_e2e:
        Ke = max(1, min(K, args.e2e_steps))
        Xh = torch.empty_like(X, device="cpu").pin_memory()
        Fh = torch.empty_like(F, device="cpu").pin_memory()
        Xh.copy_(X)
        Fh.copy_(F)
        xo = torch.empty_like(x_in, device="cpu").pin_memory()
        Ho = torch.empty_like(H, device="cpu").pin_memory()
        Yo = torch.empty_like(Y, device="cpu").pin_memory()
        chunk = min(args.e2e_chunk, T)
        ws_e2e = torch.empty(mhc.mhc_forward_host_workspace_bytes(chunk, n, d, X.dtype),
                             dtype=torch.uint8, device=dev)

        def e2e_step():
            mhc.mhc_forward_host(Xh, Fh, phi, b_pre, b_post, b_res, s["alpha_pre"], s["alpha_post"],
                                 s["alpha_res"], s["eps"], s["t_max"], xo, Ho, Yo, ws_e2e,
                                 chunk_tokens=chunk)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(Ke):
            e2e_step()
        b.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b))
        barrier()
        e2e = {"value": mdist.job_throughput(T, Ke, e_ms, world), "unit": "tokens/s",
               "h2d_bytes_per_step": (X.numel() + F.numel()) * es,
               "d2h_bytes_per_step": (x_in.numel() * es + H.numel() * 4 + Y.numel() * es),
               "steps": Ke, "api": "mhc_forward_host (pre path auto)", "chunk_tokens": chunk}
        del ws_e2e

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, seconds=args.cpu_seconds)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_total / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": workload_config(w, world, l2_bytes),
        "roofline": roofline, "hbm": hbm, "kernels": kern, "clocks": clocks, "e2e": e2e,
        "cpu_baseline": cpu, "gpu_launches": 2 * K,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward(args, rank, world, local_rank):
    """Forward + backward steps (mhc_pre_train, mhc_post, mhc_backward) on one batch: the
    backward workload (T=16384, n=4, d=4096, bf16 with outlier channels, upstream gradients
    dX_out and dx_in ~ N(0,1) in bf16).  Under torchrun every rank runs its own batch and
    the parameter gradients are all-reduced each step (data parallel).  Prints one JSON
    line."""
    import numpy as np
    import torch

    import mhc_hyper_connections_b200 as mhc
    from mhc_hyper_connections_b200 import dist as mdist
    from mhc_hyper_connections_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    w = wl.make_config(args.config)
    if args.tokens:
        w = w.tokens(np.arange(min(args.tokens, w.T)))
    T, n, d, m = w.T, w.n, w.d, w.m
    es = 2 if w.dtype == "bf16" else 4
    rng = np.random.default_rng(1000 + rank)
    up = [rng.standard_normal(sh, dtype=np.float32) for sh in ((T, n, d), (T, d))]
    if w.dtype == "bf16":
        up = [wl.bf16_round_bits(a) for a in up]

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    X, F, dY, dxi = to_dev(w.X), to_dev(w.F_out), to_dev(up[0]), to_dev(up[1])
    phi, b_pre, b_post, b_res = (to_dev(a) for a in (w.phi, w.b_pre, w.b_post, w.b_res))
    x_in = torch.empty(T, d, dtype=X.dtype, device=dev)
    H = torch.empty(T, m, device=dev)
    h = torch.empty(T, m, device=dev)
    Y = torch.empty_like(X)
    dX, dF = torch.empty_like(X), torch.empty_like(F)
    dphi = torch.empty(n * d, m, device=dev)
    db_pre, db_post, db_res = (torch.empty(n, device=dev), torch.empty(n, device=dev),
                               torch.empty(n, n, device=dev))
    dalpha = torch.empty(3, device=dev)
    ws = torch.empty(mhc.mhc_backward_workspace_bytes(T, n, d), dtype=torch.uint8, device=dev)
    s = w.scalars()
    sa = (s["alpha_pre"], s["alpha_post"], s["alpha_res"], s["eps"], s["t_max"])

    def fwd():
        mhc.mhc_pre_train(X, phi, b_pre, b_post, b_res, *sa, x_in, H, h)

    def post():
        mhc.mhc_post(X, F, H, Y)

    pgrads = dict(dphi=dphi, db_pre=db_pre, db_post=db_post, db_res=db_res, dalpha=dalpha)

    def bwd():
        mhc.mhc_backward(X, F, phi, b_pre, b_post, b_res, *sa, H, h, dY, dxi, dX, dF, dphi,
                         db_pre, db_post, db_res, dalpha, ws)
        # data-parallel step: the parameter gradients are summed over the ranks (NCCL); a
        # no-op on one GPU
        mdist.allreduce_param_grads(pgrads)

    for _ in range(args.warmup):
        fwd(); post(); bwd()
    torch.cuda.synchronize()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank)
    clk.start()
    time.sleep(0.6)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start.record()
    for k in range(K):
        e = evs[k]
        e[0].record(); fwd(); e[1].record(); post(); e[2].record(); bwd(); e[3].record()
    end.record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    time.sleep(0.3)
    clk.stop()
    ms_total = mdist.max_over_ranks(start.elapsed_time(end), device=dev)
    st = [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i in range(3)]
    value = mdist.job_throughput(T, K, ms_total, world)
    peak, peak_src = _hbm_peak()
    by_pre, by_post = bytes_per_token(n, d, es)
    by_pre += 4 * m                                            # the saved projection h
    # backward, dependency-minimal: read X, F_out, dX_out, dx_in, H, h; write dX, dF_out
    by_bwd = (3 * n + 3) * d * es + 8 * m
    bw_gbs = by_bwd * T / (st[2] / 1e3) / 1e9
    step_bytes = (by_pre + by_post + by_bwd) * T
    step_gbs = step_bytes / (ms_total / 1e3 / K) / 1e9       # per GPU: each processes T tokens
    bwd_srcs = ["mhc_hyper_connections_b200/csrc/backward.cu", "mhc_hyper_connections_b200/csrc/backward_tc.cu"]
    bwd_src = " + ".join(bwd_srcs)
    rec = NCU_TRAFFIC.get(("backward", args.config))
    traffic = rec[0] if (rec and not args.tokens and rec[1] == _src_sha(bwd_srcs)) else None
    line = {
        "metric": "mHC forward+backward tokens/s (pre_train + post + backward), n=4 d=4096 bf16",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_total / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": args.config + "+backward", "T": T, "n": n, "d": d,
                   "parallelism": f"dp{world} (token batches per rank, parameter-gradient all-reduce)",
                   "upstream": "dX_out, dx_in ~ N(0,1), stored like X",
                   "l2": "inputs larger than L2, no flush"},
        "kernels": {"pre_train": {"ms": st[0], "bytes_per_launch": by_pre * T,
                                  "gbs": by_pre * T / (st[0] / 1e3) / 1e9},
                    "post": {"ms": st[1], "bytes_per_launch": by_post * T,
                             "gbs": by_post * T / (st[1] / 1e3) / 1e9},
                    "backward": {"ms": st[2], "bytes_per_launch": by_bwd * T, "gbs": bw_gbs,
                                 "launches": 6,
                                 "source": bwd_src}},
        "roofline": {"kernel": "backward (6 launches)", "bound": "hbm", "achieved": bw_gbs,
                     "peak": peak, "unit": "GB/s", "frac": bw_gbs / peak, "traffic": traffic,
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": by_bwd * T},
        "hbm": {"step_bytes_per_token": by_pre + by_post + by_bwd, "gbs_per_gpu": step_gbs,
                "frac_of_peak": step_gbs / peak, "peak_source": peak_src},
        "clocks": clk.summary(t_wall0, t_wall1), "e2e": None, "cpu_baseline": None,
        "gpu_launches": 8 * K,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_amax(args, rank, world, local_rank):
    """The depth-stability diagnostic: mhc_amax_gain over the coefficient rows of L = 60
    layers (the 27B model's depth) for T tokens at n = 4.  Prints one JSON line."""
    import torch

    import mhc_hyper_connections_b200 as mhc
    from mhc_hyper_connections_b200 import dist as mdist
    from mhc_hyper_connections_b200 import workloads as wl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = wl.make_config(args.config)
    T = args.tokens or w.T
    n, L = w.n, 60
    m = n * n + 2 * n
    g = torch.Generator(device=dev)
    g.manual_seed(1234 + rank)
    Hs = torch.rand(L, T, m, device=dev, generator=g)          # stand-in maps, fp32
    gain = torch.empty(L, T, 2, device=dev)
    for _ in range(args.warmup):
        mhc.mhc_amax_gain(Hs, gain)
    torch.cuda.synchronize()
    K = args.steps
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(K):
        mhc.mhc_amax_gain(Hs, gain)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    ms = mdist.max_over_ranks(ms, device=dev)
    by = L * T * (m * 4 + 8)
    peak, peak_src = _hbm_peak()
    gbs = by / (ms / 1e3 / K) / 1e9
    line = {"metric": "mHC composite Amax gain (diagnostic): layer-tokens/s, L=60 n=4",
            "value": L * T * K * world / (ms / 1e3), "unit": "layer-tokens/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"amax_L{L}_T{T}_n{n}", "L": L, "T": T, "n": n},
            "roofline": {"kernel": "amax_gain_kernel", "bound": "hbm", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak, "traffic": None, "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": by},
            "gpu_launches": K}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    from mhc_hyper_connections_b200 import workloads as wl
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=wl.HEADLINE, choices=sorted(wl.CONFIGS))
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T of the workload (smaller cases for profiling)")
    ap.add_argument("--pre-path", default="auto",
                    choices=["auto", "generic", "cluster_tc", "two_pass_tc"],
                    help="kernel path of the pre stage (default: the library's choice)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-chunk", type=int, default=1024,
                    help="tokens per chunk of the end-to-end mhc_forward_host call")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--amax", action="store_true",
                    help="time the composite Amax gain diagnostic (mhc_amax_gain, 60 layers)")
    ap.add_argument("--backward", action="store_true",
                    help="time forward + backward steps (mhc_pre_train, mhc_post, mhc_backward)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 needs one process per GPU (torchrun --nproc-per-node N)")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.backward:
        return run_backward(args, rank, world, local_rank)
    if args.amax:
        return run_amax(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
