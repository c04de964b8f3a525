#!/usr/bin/env python
"""Benchmark of the chunkwise gated delta rule on B200: one JSON line on rank 0.

A step is one pass of the whole path over one batch of synthetic input: the
forward (o, u, S_T) and the backward (dq, dk, dv, d log alpha, dbeta, dS0) of
Gated DeltaNet at B=8, T=4096, H=8, dk=dv=128, bf16 I/O, fp32 state, chunk 64
(the headline workload "delta-rule fwd+bwd tokens/s at B=8,T=4096,H=8,d=128
bf16").  Inputs are drawn once by the seeded generator and are resident in HBM
before the timed region.  Each step is timed with CUDA events on the launching
stream; L2 is flushed (256 MiB write) between steps, outside the events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs an independent replica
(the path has no cross-(b, h) exchange, so there is no data-path collective);
value = all ranks' tokens / the slowest rank's time ("scaling": "weak").

--impl reference times the fp64 CPU oracle (the checker, test infrastructure) on
a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "delta-rule fwd+bwd tokens/s at B=8,T=4096,H=8,d=128 bf16; % of roofline"
WORKLOAD_ID = 2
DECODE_B = 64  # sequences in the decoding-step measurement
FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------------------------
# algorithmic counts (per token-head unless stated)
def alg_counts(B, T, H, dk, dv, C, variant, elem, s0=False, du=True):
    gw = {0: 0, 1: 1, 2: dk}[variant]
    th = B * T * H
    heads = B * H
    fwd_flops = th * (6 * dk * dv + 3 * C * dk + 2 * C * dv + C * C / 3)
    fwd_bytes = th * elem * (2 * dk + 3 * dv + gw + 1) + heads * 4 * dk * dv * (1 + int(s0))
    bwd_in_out = (4 * dk + 4 * dv + 2 * gw + 2) - (0 if du else dv)
    bwd_bytes = th * elem * bwd_in_out + heads * 4 * dk * dv * (2 + int(s0))
    return {"fwd_flops": fwd_flops, "fwd_bytes": fwd_bytes, "bwd_flops": 2 * fwd_flops, "bwd_bytes": bwd_bytes,
            # the per-token-head backward inputs and outputs, without the per-head states
            "bwd_io_bytes": th * elem * bwd_in_out,
            # what the intra-chunk gradient kernel itself reads and writes: the same without du,
            # which the reverse chain consumes (it hands the kernel dL/dU instead)
            "bwd_grad_kernel_bytes": th * elem * (bwd_in_out - (dv if du else 0))}


def workload_config(w, B, world):
    """The config object of the JSON line; both arms print the same one."""
    name = w.name if B == w.B else w.name.replace(f"_B{w.B}_", f"_B{B}_")
    return {"workload": name + " fwd+bwd", "B": B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv, "chunk": 64,
            "variant": {0: "deltanet", 1: "gdn", 2: "kda"}[w.variant], "io": "bf16, fp32 state",
            "l2": "flushed between steps (256 MiB write)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.proc = None
        self.lines = []
        self.uuid = device_uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
def cpu_oracle_sample(w, steps=1, seed=0):
    """Time the fp64 oracle (fwd + bwd) on a bounded sample of the workload.

    The sample is `units` (b, h) sequences of the full length T (one per host
    core, the oracle's own threading unit), drawn by the same generator.  The
    rate is extrapolated to the whole workload by the (b, h) count.
    """
    import numpy as np
    import torch

    import oracle
    from gated_delta_rule_107_b200.inputs import make_inputs

    cores = os.cpu_count() or 1
    units = max(1, min(cores, w.B * w.H))
    x = make_inputs(w.variant, w.dtype, 1, w.T, units, w.dk, w.dv, seed=w.seed + 77, grads=True, du=True)
    a = {k: (None if v is None else v.double().numpy()) for k, v in x.items()}
    oracle.load_library()
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle.fwd(a["q"], a["k"], a["v"], a["loga"], a["beta"], None, variant=w.variant, nthreads=units)
        oracle.bwd(a["q"], a["k"], a["v"], a["loga"], a["beta"], None, a["dO"], a["du"], a["dS_T"],
                   variant=w.variant, nthreads=units)
        times.append(time.perf_counter() - t0)
    t = statistics.median(times)
    full_time = t * (w.B * w.H) / units
    value = w.B * w.T / full_time
    sample = (f"fp64 oracle fwd+bwd on {units} (b,h) sequences of T={w.T} (of {w.B * w.H}); "
              f"{t:.2f} s per sample; the rate is extrapolated to the workload by the (b,h) count")
    return {"value": value, "unit": "tokens/s", "cores": units, "kind": "oracle", "sample": sample,
            "sample_seconds": t}, times, np


# ---------------------------------------------------------------------------------------------
# Replicas (N > 1, one rank per GPU): every rank solves its own independent (b, h) problems --
# the path has no exchange step -- and the job's time is the slowest rank's.
def replica_seed(seed: int, rank: int) -> int:
    """Seed of a rank's replica: each rank draws its own inputs."""
    return seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over the ranks of the default process group (x itself alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, world: int, ms_max: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_107_b200.inputs import WORKLOADS
    w = WORKLOADS[WORKLOAD_ID]
    cpu_oracle_sample(w, steps=max(args.warmup, 0) or 1)  # warm-up
    base, times, _ = cpu_oracle_sample(w, steps=args.steps)
    ms_sample = statistics.mean(times) * 1e3  # one step as run: the bounded sample
    line = {
        "impl": "reference", "metric": METRIC, "value": base["value"], "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_sample, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, w.B, 1),
        "step": f"the fp64 oracle (fwd + bwd) on {base['cores']} of the workload's {w.B * w.H} (b,h) sequences, "
                "full length, one thread each",
        "ms_per_step_whole_workload_extrapolated": ms_sample * (w.B * w.H) / base["cores"],
        "cpu_baseline": base,
        "e2e": {"value": base["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    from gated_delta_rule_107_b200 import binding
    from gated_delta_rule_107_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (B200); the CPU oracle arm is --impl reference")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = WORKLOADS[args.workload]
    B, T, H, dk, dv, C, var = (args.batch or w.B), w.T, w.H, w.dk, w.dv, 64, w.variant
    vname = {0: "deltanet", 1: "gdn", 2: "kda"}[var]
    dt = binding.DR_BF16
    x = make_inputs(var, w.dtype, B, T, H, dk, dv, seed=replica_seed(w.seed, rank), s0_std=w.s0_std, grads=True, du=True,
                    device=dev)
    s0 = x["S0"] if w.s0_std else None
    elem = 2

    # The timed step is the training pair: the forward keeps what the backward would
    # recompute (delta_rule_fwd_save), the backward starts from it (delta_rule_bwd_saved).
    # The plain forward + recomputing backward is timed afterwards and reported beside it.
    sv_bytes = binding.saved_size(B, T, H, dk, dv, var, C, dt)
    saved = torch.empty(max(sv_bytes, 1), dtype=torch.uint8, device=dev)
    ws_bytes = max(binding.workspace_size(B, T, H, dk, dv, var, C, dt, kind) for kind in range(4))
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    o = torch.empty_like(x["v"])
    u = torch.empty_like(x["v"])
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    grads = {"dq": torch.empty_like(x["q"]), "dk": torch.empty_like(x["k"]), "dv": torch.empty_like(x["v"]),
             "dalpha": torch.empty_like(x["loga"]), "dbeta": torch.empty_like(x["beta"]),
             "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)}
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731

    def make_step(saved_pair: bool):
        fk, bk = (2, 3) if saved_pair else (0, 1)
        fnames = binding.launches(B, T, H, dk, dv, var, C, dt, fk)
        bnames = binding.launches(B, T, H, dk, dv, var, C, dt, bk)
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(len(fnames) + 1)]
        be = [torch.cuda.Event(enable_timing=True) for _ in range(len(bnames) + 1)]
        for e in fe + be:  # torch creates the CUDA event handle on first record
            e.record(stream)
        torch.cuda.synchronize()
        fa_ev, ba_ev = binding.event_array(fe), binding.event_array(be)
        fa = (p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(s0), p(o), p(u), p(S_T),
              B, T, H, dk, dv, var, C, dt)
        ba = (p(x["q"]), p(x["k"]), p(x["v"]), p(x["loga"]), p(x["beta"]), p(s0), p(x["dO"]), p(x["du"]),
              p(x["dS_T"]), p(grads["dq"]), p(grads["dk"]), p(grads["dv"]), p(grads["dalpha"]), p(grads["dbeta"]),
              p(grads["dS0"]), B, T, H, dk, dv, var, C, dt)
        sv = (p(saved), sv_bytes)
        wsa = (p(ws), ws_bytes, sp)

        def step(timed: bool, mid=None):
            # timed: the calls that record an event between every two kernels; mid: an event
            # recorded between the forward and the backward call
            if saved_pair and timed:
                rc1 = binding.fwd_save_timed_raw(*fa, *sv, *wsa, fa_ev, len(fe))
                rc2 = binding.bwd_saved_timed_raw(*ba, *sv, *wsa, ba_ev, len(be))
            elif saved_pair:
                rc1 = binding.fwd_save_raw(*fa, *sv, *wsa)
                if mid is not None:
                    mid.record()
                rc2 = binding.bwd_saved_raw(*ba, *sv, *wsa)
            elif timed:
                rc1 = binding.fwd_timed_raw(*fa, *wsa, fa_ev, len(fe))
                rc2 = binding.bwd_timed_raw(*ba, *wsa, ba_ev, len(be))
            else:
                rc1 = binding.fwd_raw(*fa, *wsa)
                if mid is not None:
                    mid.record()
                rc2 = binding.bwd_raw(*ba, *wsa)
            if rc1 or rc2:
                raise RuntimeError(f"delta_rule call failed: {binding.strerror(rc1 or rc2)}")

        return step, fnames, bnames, fe, be

    step, fwd_names, bwd_names, fev, bev = make_step(True)

    for _ in range(max(args.warmup, 3)):
        step(False)
    torch.cuda.synchronize()
    if binding.sync_status() != binding.DR_OK:
        raise RuntimeError("device error word set during warm-up")

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    t_pre = time.perf_counter()
    while time.perf_counter() - t_pre < 0.4:  # load the GPU before the first sample
        step(False)
        torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # The timed steps: the two calls as a user makes them, with an event before, between and after
    # them (L2 flushed before each step).  Then the same number of steps again through the calls
    # that record an event between every two kernels, for the per-kernel times; those events
    # lengthen a step (by about 1.6 % at the headline shape), so the step time is the first pass's.
    ea, em, eb = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    step_ms, fwd_ms, bwd_ms = [], [], []
    for _ in range(args.steps):
        flush.fill_(1)
        ea.record()
        step(False, mid=em)
        eb.record()
        torch.cuda.synchronize()
        step_ms.append(ea.elapsed_time(eb))
        fwd_ms.append(ea.elapsed_time(em))
        bwd_ms.append(em.elapsed_time(eb))
    torch.cuda.synchronize()
    kern, inst_ms = {n: [] for n in set(fwd_names) | set(bwd_names)}, []
    for _ in range(args.steps):
        flush.fill_(1)
        step(True)
        torch.cuda.synchronize()
        fms = [fev[i].elapsed_time(fev[i + 1]) for i in range(len(fwd_names))]
        bms = [bev[i].elapsed_time(bev[i + 1]) for i in range(len(bwd_names))]
        for n, t in zip(fwd_names, fms):
            kern[n].append(t)
        for n, t in zip(["bwd:" + n for n in bwd_names], bms):
            kern.setdefault(n, []).append(t)
        inst_ms.append(fev[0].elapsed_time(fev[-1]) + bev[0].elapsed_time(bev[-1]))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    if binding.sync_status() != binding.DR_OK:
        raise RuntimeError("device error word set during the timed region")

    ms = max_over_ranks(statistics.mean(step_ms), dev)
    tokens = B * T * world
    value = weak_scaling_value(B * T, world, ms)

    # ---- the plain forward + recomputing backward, same protocol (reported beside) ----
    rstep, rf_names, rb_names, rfev, rbev = make_step(False)
    for _ in range(max(args.warmup, 3)):
        rstep(False)
    torch.cuda.synchronize()
    r_plain = []  # the two calls as a user makes them, then the same steps with per-kernel events
    for _ in range(args.steps):
        flush.fill_(1)
        ea.record()
        rstep(False)
        eb.record()
        torch.cuda.synchronize()
        r_plain.append(ea.elapsed_time(eb))
    r_kern = {}
    for _ in range(args.steps):
        flush.fill_(1)
        rstep(True)
        torch.cuda.synchronize()
        for n, i in zip(rf_names, range(len(rf_names))):
            r_kern.setdefault(n, []).append(rfev[i].elapsed_time(rfev[i + 1]))
        for n, i in zip(rb_names, range(len(rb_names))):
            r_kern.setdefault("bwd:" + n, []).append(rbev[i].elapsed_time(rbev[i + 1]))
    if binding.sync_status() != binding.DR_OK:
        raise RuntimeError("device error word set during the recompute leg")
    r_ms = max_over_ranks(statistics.mean(r_plain), dev)

    # ---- one decoding step (delta_rule_decode), reported beside: DECODE_B sequences, one
    # token each, the fp32 state updated in place; L2 flushed before every call ----
    dx = make_inputs(var, "bf16", DECODE_B, 1, H, dk, dv, seed=w.seed + 7, s0_std=0.05, device=dev)
    dS = dx["S0"]
    dev_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for _ in range(3):
        binding.delta_rule_decode(dx["q"], dx["k"], dx["v"], dx["loga"], dx["beta"], dS, variant=var, inplace=True)
    dec_ms = []
    for _ in range(args.steps):
        flush.fill_(1)
        dev_ev[0].record()
        binding.delta_rule_decode(dx["q"], dx["k"], dx["v"], dx["loga"], dx["beta"], dS, variant=var, inplace=True)
        dev_ev[1].record()
        torch.cuda.synchronize()
        dec_ms.append(dev_ev[0].elapsed_time(dev_ev[1]))
    if binding.sync_status() != binding.DR_OK:
        raise RuntimeError("device error word set during the decode leg")
    d_ms = statistics.mean(dec_ms)
    g_w = {binding.DR_DELTANET: 0, binding.DR_GATED: 1, binding.DR_KDA: dk}[var]
    d_bytes = DECODE_B * H * (2 * 4 * dk * dv + elem * (2 * dk + 3 * dv + g_w + 1))
    decode = {"workload": f"{vname} decode bf16 B{DECODE_B} T1 H{H} d{dk}, fp32 state updated in place",
              "ms_per_step": d_ms, "tokens_per_s": DECODE_B / (d_ms / 1e3), "alg_bytes": d_bytes,
              "roofline": {"bound": "hbm", "achieved": d_bytes / (d_ms / 1e3) / 1e9, "unit": "GB/s",
                           "frac": d_bytes / (d_ms / 1e3) / 1e9 / load_peaks()["hbm_gbs"]},
              "kernel": "k_decode"}

    # ---- the single-pass operations around the core at this shape, reported beside ----
    def ev_time(fn, reps=5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.mean(ts)

    gw_ = 0 if var == binding.DR_DELTANET else (dk if var == binding.DR_KDA else 1)
    rows = B * T * H
    raw_a = None if var == binding.DR_DELTANET else torch.randn_like(x["loga"].float()).to(x["q"].dtype) - 3.0
    pre_out = binding.delta_rule_preop(x["q"], x["k"], x["beta"], raw_a, variant=var)
    pre_ms = ev_time(lambda: binding.delta_rule_preop(x["q"], x["k"], x["beta"], raw_a, variant=var))
    pre_b_ms = ev_time(lambda: binding.delta_rule_preop_bwd(x["q"], x["k"], x["beta"], raw_a, pre_out[0], pre_out[1],
                                                            pre_out[2], pre_out[3], variant=var))
    post_w = torch.ones(dv, device=dev)
    post_ms = ev_time(lambda: binding.delta_rule_postop(o, u, post_w))
    post_b_ms = ev_time(lambda: binding.delta_rule_postop_bwd(o, u, post_w, x["dO"]))
    # cross-layer routing of this step's write values into a hidden stream of H*dv channels
    n_hid = H * dv
    clvr_W = (0.05 * torch.randn(H * dv, n_hid, device=dev)).to(u.dtype)
    clvr_h = torch.randn(B, T, n_hid, device=dev).to(u.dtype)
    clvr_ws = torch.empty(binding.load().delta_rule_clvr_workspace_size(), dtype=torch.uint8, device=dev)
    clvr_ms = ev_time(lambda: binding.delta_rule_clvr(u, clvr_W, clvr_h, workspace=clvr_ws))
    clvr_b_ms = ev_time(lambda: binding.delta_rule_clvr_bwd(u, clvr_W, clvr_h, workspace=clvr_ws))
    conv_w = 0.5 * torch.randn(H * dk, 4, device=dev)
    conv_ms = ev_time(lambda: binding.delta_rule_shortconv(x["q"], conv_w))
    conv_b_ms = ev_time(lambda: binding.delta_rule_shortconv_bwd(x["q"], conv_w, x["q"]))
    if binding.sync_status() != binding.DR_OK:
        raise RuntimeError("device error word set during the pre/post leg")
    pre_unit = rows * elem * (2 * dk + 1 + gw_)  # q, k, beta, gate of every row once
    post_bytes = rows * elem * 3 * dv
    hbm = load_peaks()["hbm_gbs"]

    def gbs(nbytes, t_ms):
        return {"ms": t_ms, "alg_bytes": nbytes, "achieved_gbs": nbytes / (t_ms / 1e3) / 1e9,
                "frac": nbytes / (t_ms / 1e3) / 1e9 / hbm}

    prepost = {"shape": f"B{B} T{T} H{H} d{dk} bf16", "preop": gbs(2 * pre_unit, pre_ms),
               "preop_bwd": gbs(3 * pre_unit, pre_b_ms), "postop": gbs(post_bytes, post_ms),
               "postop_bwd": gbs(rows * elem * 5 * dv, post_b_ms),
               # one [B, T, H*dk] stream: x read, y written (backward: x, dy read, dx written)
               "shortconv": gbs(2 * rows * elem * dk, conv_ms), "shortconv_bwd": gbs(3 * rows * elem * dk, conv_b_ms)}

    # the fused forward (pre-operation, forward and post-operation in the core's own kernels)
    # against the three separate calls, on the same raw inputs (Gated DeltaNet / DeltaNet only)
    fused = None
    if var != binding.DR_KDA:
        go_ = torch.randn_like(x["v"].float()).to(x["v"].dtype)
        w_ = torch.ones(dv, device=dev)
        fws = torch.empty(binding.fused_workspace_size(B, T, H, dk, dv, var, C, binding.DR_BF16), dtype=torch.uint8,
                          device=dev)
        fused_ms = ev_time(lambda: binding.delta_rule_fwd_fused(x["q"], x["k"], x["v"], raw_a, x["beta"], go_, w_,
                                                                 variant=var, workspace=fws))

        def three():
            q_, k_, b_, a_ = binding.delta_rule_preop(x["q"], x["k"], x["beta"], raw_a, variant=var)
            o_, _, _ = binding.delta_rule_fwd(q_, k_, x["v"], a_, b_, None, variant=var)
            binding.delta_rule_postop(o_, go_, w_)

        three_ms = ev_time(three)
        if binding.sync_status() != binding.DR_OK:
            raise RuntimeError("device error word set during the fused leg")
        f_alg = rows * elem * (2 * dk + 2 * dv + gw_ + 1 + 2 * dv)  # raw q, k, v, gate, beta, out gate in; y, u out
        fused = {"shape": f"B{B} T{T} H{H} d{dk} bf16", "fused_ms": fused_ms, "separate_ms": three_ms,
                 "saved_ms": three_ms - fused_ms, "kernels": ["k_chunk_prep(raw)", "k_chain_fwd(fused, 2-CTA clusters)"],
                 "alg_bytes": f_alg, "fused_frac": f_alg / (fused_ms / 1e3) / 1e9 / hbm}

    clvr_flops = 2.0 * B * T * (H * dv) * n_hid
    bf16_peak = load_peaks().get("bf16_tflops")
    clvr = {"shape": f"M{B * T} K{H * dv} N{n_hid} bf16 (k_gemm_tc)", "fwd_ms": clvr_ms, "bwd_ms": clvr_b_ms,
            "fwd_tflops": clvr_flops / (clvr_ms / 1e3) / 1e12, "bwd_tflops": 2 * clvr_flops / (clvr_b_ms / 1e3) / 1e12}
    if bf16_peak:
        clvr["fwd_frac"] = clvr["fwd_tflops"] / bf16_peak
        clvr["bwd_frac"] = clvr["bwd_tflops"] / bf16_peak

    # ---- end to end through the public API with host buffers ----
    # Every step copies its inputs in from pinned host memory and its results out to pinned host
    # memory.  The copies in, the two calls and the copies out run on three streams with two sets
    # of device buffers, so that step i's inputs travel while step i - 1 computes and step i - 2's
    # results travel back (PCIe carries both directions at once); events order each buffer's
    # reuse.
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in x.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    out_sets = [{"o": o, "u": u, "S_T": S_T, "grads": grads},
                {"o": torch.empty_like(o), "u": torch.empty_like(u), "S_T": torch.empty_like(S_T),
                 "grads": {k: (torch.empty_like(v) if v is not None else None) for k, v in grads.items()}}]

    def out_list(os_):
        return [os_["o"], os_["u"], os_["S_T"]] + [g for g in os_["grads"].values() if g is not None]

    d2h = sum(t.numel() * t.element_size() for t in out_list(out_sets[0]))
    host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in out_list(os_)] for os_ in out_sets]
    in_sets = [{k: (torch.empty_like(v) if v is not None else None) for k, v in x.items()} for _ in range(2)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in_free", "in_ready", "out_ready", "out_free")}

    def e2e_step(i):
        j = i % 2
        din, os_ = in_sets[j], out_sets[j]
        s_in.wait_event(ev["in_free"][j])
        with torch.cuda.stream(s_in):
            for k_, v_ in host.items():
                if v_ is not None:
                    din[k_].copy_(v_, non_blocking=True)
        ev["in_ready"][j].record(s_in)
        s_cmp.wait_event(ev["in_ready"][j])
        s_cmp.wait_event(ev["out_free"][j])
        with torch.cuda.stream(s_cmp):
            s0_in = din["S0"] if s0 is not None else None
            _, _, _, sv = binding.delta_rule_fwd_save(din["q"], din["k"], din["v"], din["loga"], din["beta"], s0_in,
                                                      variant=var, chunk=C, saved=saved, workspace=ws, out=os_["o"],
                                                      u=os_["u"], S_T=os_["S_T"])
            binding.delta_rule_bwd_saved(din["q"], din["k"], din["v"], din["loga"], din["beta"], s0_in, din["dO"],
                                         din["du"], din["dS_T"], saved=sv, variant=var, chunk=C, workspace=ws,
                                         grads=os_["grads"])
        ev["in_free"][j].record(s_cmp)
        ev["out_ready"][j].record(s_cmp)
        s_out.wait_event(ev["out_ready"][j])
        with torch.cuda.stream(s_out):
            for src, dst in zip(out_list(os_), host_out[j]):
                dst.copy_(src, non_blocking=True)
        ev["out_free"][j].record(s_out)

    e2e_ms = float("nan")
    if not args.no_e2e:
        main = torch.cuda.current_stream(dev)
        for j in range(2):
            ev["in_free"][j].record(main)
            ev["out_free"][j].record(main)
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(3, min(args.steps, 10))
        e0.record(main)
        for s_ in (s_in, s_cmp, s_out):
            s_.wait_stream(main)
        for i in range(e2e_steps):
            e2e_step(i)
        for s_ in (s_in, s_cmp, s_out):
            main.wait_stream(s_)
        e1.record(main)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        if binding.sync_status() != binding.DR_OK:
            raise RuntimeError("device error word set during the end-to-end leg")

    peaks = load_peaks()
    cnt = alg_counts(B, T, H, dk, dv, C, var, elem, s0=s0 is not None)
    kern_ms = {n: statistics.mean(v) for n, v in kern.items() if v}
    total = sum(kern_ms.values())
    dominant = max(kern_ms, key=kern_ms.get)
    f_ms = statistics.mean(fwd_ms)
    b_ms = statistics.mean(bwd_ms)
    # Roofline of the gradient kernel (the largest share of the step): it reads the backward
    # inputs q, k, v, beta, the gate and dO and writes every backward output (dq, dk, dv, dbeta,
    # d log alpha), so its algorithmic bytes per launch are those per-token-head counts times
    # B*T*H; du goes to the reverse chain (which hands the kernel dL/dU), and so do the states
    # dS_T / dS0.
    rk = "bwd:k_bwd_chunk_tc"
    if rk not in kern_ms:  # another path (e.g. KDA): the whole backward call
        rk = None
    r_bytes = cnt["bwd_grad_kernel_bytes"] if rk else cnt["bwd_bytes"]
    rk_ms = kern_ms[rk] if rk else b_ms
    achieved = r_bytes / (rk_ms / 1e3) / 1e9
    r_label = rk.split(":", 1)[1] if rk else "backward call (" + "+".join(bwd_names) + ")"
    # the forward call at T = 4096 against its own algorithmic bytes
    f_bytes = cnt["fwd_bytes"]
    f_achieved = f_bytes / (f_ms / 1e3) / 1e9
    fwd_label = fwd_names[0] if len(fwd_names) == 1 else "forward call (" + "+".join(fwd_names) + ")"
    traffic = None
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        try:
            from gated_delta_rule_107_b200.build import source_digest
            with open(tfile) as f:
                tr = json.load(f)
            ent = tr.get(r_label)
            # counters stay valid while the files that define the kernel are unchanged
            if ent and ent.get("source_digest") == source_digest(ent.get("source_files")):
                traffic = ent["bytes_per_launch"] * (B / ent.get("batch", B))
        except Exception:
            traffic = None
    step_time_roof = max((cnt["fwd_bytes"] + cnt["bwd_bytes"]) / (peaks["hbm_gbs"] * 1e9),
                         (cnt["fwd_flops"] + cnt["bwd_flops"]) / (peaks["bf16_tflops_sustained"] * 1e12))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, B, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": r_label,
                     "alg_bytes_per_launch": r_bytes, "ms_per_launch": rk_ms,
                     "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs, burst copy)"},
        "fwd_roofline": {"bound": "hbm", "achieved": f_achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": f_achieved / peaks["hbm_gbs"], "kernel": fwd_label, "alg_bytes_per_call": f_bytes,
                         "ms_per_call": f_ms},
        "step_roofline": {"alg_bytes": cnt["fwd_bytes"] + cnt["bwd_bytes"],
                          "alg_flops": cnt["fwd_flops"] + cnt["bwd_flops"], "roofline_ms": step_time_roof * 1e3,
                          "frac": step_time_roof * 1e3 / ms, "fwd_ms": f_ms, "bwd_ms": b_ms},
        "kernels": {n: {"ms": round(t, 4), "share": round(t / total, 4)} for n, t in kern_ms.items()},
        "instrumented_ms_per_step": statistics.mean(inst_ms),  # the same steps with an event between kernels
        "dominant_kernel": dominant,
        "step": "delta_rule_fwd_save + delta_rule_bwd_saved (the forward keeps the chunk products and states the "
                "backward reads; every value is computed inside the timed step)",
        "recompute": {"step": "delta_rule_fwd + delta_rule_bwd (the backward recomputes the forward)",
                      "ms_per_step": r_ms, "value": tokens / (r_ms / 1e3),
                      "kernels": {n: round(statistics.mean(v), 4) for n, v in r_kern.items()}},
        "saved_bytes": sv_bytes,
        "decode": decode,
        "prepost": prepost,
        "fused": fused,
        "clvr": clvr,
        # the timed steps' kernels: the plain calls' launches (more when they run in segments)
        "gpu_launches": args.steps * (binding.plain_launches(B, T, H, dk, dv, var, C, dt, 2)
                                      + binding.plain_launches(B, T, H, dk, dv, var, C, dt, 3)),
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "overlap": "copies in, compute and copies out on three streams, two buffer sets across steps"},
        "clocks": clocks,
        "gpu": torch.cuda.get_device_name(dev),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w, steps=1)[0]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload at this batch size instead (smaller cases for ncu captures)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--workload", type=int, default=WORKLOAD_ID, choices=(2, 3, 4, 5),
                    help="workload id (default: the headline GDN B=8 T=4096 H=8 d=128; 3-5 are the other bf16 ones)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
