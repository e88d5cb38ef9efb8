#!/usr/bin/env python3
"""Benchmark of DeltaLog decode on B200: one JSON line on rank 0.

A step is one merge cycle of an R-layer stack of identical decode layers:
C tokens, each through all R layers in turn -- C-1 append + read-out steps
and one merge-token step per layer -- as one CUDA-graph launch
(dl_cycle_launch).  R rotating layers keep every base read cold in L2
(working set >= 4x the 126 MB L2).  Throughput is decode tokens per second
through one layer (B sequences x C tokens x R layers per step), the
amortised latency is the step time / (C R).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--layers R] [--impl native|reference]

Under torchrun (N > 1) every rank runs its own replica (independent
batches, no collective on the data path); rank 0 prints the aggregate with
the time taken as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = ("amortized µs/token state update, decode tok/s, HBM GB/s vs roofline, "
          "bytes written/token")
DEFAULT_WORKLOAD = "gdn-b128-h16-d128-c8"
L2_BYTES = 126 * 1000 * 1000
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "source": "fallback"}


# ------------------------------------------------------------ ranks ------

def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world, backend, timeout_s=120):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def reduce_over_ranks(elapsed_ms: float, units: float, device=None):
    """(max elapsed over ranks, sum of units over ranks); identity at N = 1."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(elapsed_ms), float(units)
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------ byte model ------

def bytes_model(w, fold=True):
    """Algorithmic HBM bytes per head (read, write) of each kernel.

    append(L): base read once, L logged entries (key, value factor,
    log-decay), the token's inputs; writes the output and one log entry.
    merge_token(L): base read and written, L entries, inputs read, output
    written.  merge(L): base read + L entries, base written.  eager: state
    read and written, inputs read, output written.  A merge cycle of C
    tokens is C-1 appends + a merge-token (fold) or C appends + a merge."""
    ie = 2 if w.in_dtype == "bf16" else 4
    oe = 2 if w.out_dtype == "bf16" else 4
    ue = ie if w.op == 2 else 4
    m = w.m
    S = 4 * w.dk * w.dv
    E = w.dk * ie + w.dv * ue + 4 * m
    I = (2 * w.dk + w.dv) * ie + 4 * m + (0 if w.op == 2 else 4) + (4 * w.dk if w.op == 2 else 0)
    O = w.dv * oe

    def append(L):
        return S + L * E + I, O + E

    def merge_token(L):
        return S + L * E + I, S + O

    def merge(L):
        return S + L * E, S

    eager = (S + I, S + O)
    C = w.C
    if fold:
        cyc = [append(L) for L in range(C - 1)] + [merge_token(C - 1)]
    else:
        cyc = [append(L) for L in range(C)] + [merge(C)]
    return {"S": S, "E": E, "I": I, "O": O, "append": append, "merge": merge,
            "merge_token": merge_token, "eager": eager,
            "token_read": sum(r for r, _ in cyc) / C, "token_write": sum(x for _, x in cyc) / C}


# --------------------------------------------------------- clocks -------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread.
    Entering waits (at most a second) for the thread's first sample, so
    that a short timed region that follows is sampled from its start."""

    def __init__(self, torch_device, period_s=0.001):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.h = None
        self._stop = threading.Event()
        self._first = threading.Event()
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            props = __import__("torch").cuda.get_device_properties(torch_device)
            h = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    h = N.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                except Exception:
                    h = None
            if h is None:
                h = N.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.h = h
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = repr(e)

    def _run(self):
        N = self.N
        fn = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            N.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM),
                                     int(fn(self.h))))
            except Exception:
                pass
            self._first.set()
            self._stop.wait(self.period)

    def __enter__(self):
        if self.h is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            self._first.wait(1.0)
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.h is not None:
            self.t.join()

    def summary(self):
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": getattr(self, "error", "nvml unavailable")}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        reasons = set()
        for _, r in busy:
            for bit, name in _REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    except Exception:
        return dict(PEAKS_FALLBACK)


def kernel_source_digest(path):
    """sha256 of a CUDA source with its comments and blank space removed, so
    that it changes exactly when the code does."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = " ".join(text.split())
    return hashlib.sha256(text.encode()).hexdigest()


def recorded_traffic(workload_name):
    """Per-launch DRAM bytes of the append kernel from the committed ncu
    summary, if it was taken on the current kernel code (else None)."""
    path = os.path.join(ROOT, "profiles", f"append_kernel_{workload_name}.md")
    src = os.path.join(ROOT, "recurrent_state_head_b200", "csrc", "kernels.cuh")
    try:
        text = open(path).read()
        sha = kernel_source_digest(src)
        m_sha = re.search(r"kernel_code_sha256:\s*([0-9a-f]{64})", text)
        m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        if m_sha and m_b and m_sha.group(1) == sha:
            return float(m_b.group(1))
    except OSError:
        pass
    return None


# ------------------------------------------------------- CPU oracle -----

def cpu_oracle_sample(w, target_s=12.0, seed=99, extras=True):
    """Time the fp64 oracle's base+log decode on a bounded sample of the
    workload -- a random subset of its heads over whole merge cycles -- sized
    to about `target_s` seconds of host work.  Returns tok/s in the GPU's
    unit (head-tokens per second / H), the threads used and the sample."""
    import oracle
    from recurrent_state_head_b200 import synth

    threads = max(1, len(os.sched_getaffinity(0)))
    rng = np.random.default_rng(seed)
    S_all = synth.initial_state(w).reshape(w.heads, w.dk, w.dv)
    bon_all = synth.bonus(w)

    def run(n_heads, n_cycles, n_threads=threads, eager=False):
        heads = np.sort(rng.choice(w.heads, size=min(n_heads, w.heads), replace=False))
        T = n_cycles * w.C
        ti = synth.tokens(w, 0, T, heads=heads)
        g = ti.g.astype(np.float64)
        if g.ndim == 2:
            g = g[:, :, None]
        bon = None if bon_all is None else bon_all[heads % w.H]
        beta = None if w.op == 2 else ti.beta.astype(np.float64)
        t0 = time.perf_counter()
        if eager:
            oracle.eager_run(w.op, S_all[heads], ti.q64, ti.k64, ti.v64, beta, g, bon, w.scale,
                             n_threads=n_threads)
        else:
            st = oracle.LogState(w.op, S_all[heads], w.C)
            oracle.deltalog_run(st, ti.q64, ti.k64, ti.v64, beta, g, bon, w.scale,
                                n_threads=n_threads)
        return time.perf_counter() - t0, len(heads), T

    probe = min(w.heads, max(4 * threads, 16))
    dt, n, T = run(probe, 1)
    per_head_token = dt / (n * T)
    budget = target_s / max(per_head_token, 1e-9)            # head-tokens to run
    n_heads = int(min(w.heads, max(probe, budget / w.C)))
    n_cycles = int(max(1, min(w.T // w.C, budget / (n_heads * w.C))))
    dt, n, T = run(n_heads, n_cycles)
    out = {"value": n * T / dt / w.H, "unit": "tok/s", "cores": threads, "kind": "oracle",
           "sample": f"{n} of {w.heads} heads x {T} tokens ({n_cycles} merge cycles), "
                     f"fp64 base+log oracle, {dt:.1f} s on {threads} threads"}
    if not extras:
        return out
    # one thread, and the eager recurrence on all threads, on smaller samples
    h1 = max(1, min(n_heads, int(0.15 * target_s / max(per_head_token * threads * w.C, 1e-9))))
    dt1, n1, T1 = run(h1, 1, n_threads=1)
    dte, ne, Te = run(n_heads, 1, eager=True)
    out.update({"value_1thread": n1 * T1 / dt1 / w.H,
                "eager_value": ne * Te / dte / w.H,
                "extra_samples": f"1 thread: {n1} heads x {T1} tokens in {dt1:.1f} s; eager: {ne} heads "
                                 f"x {Te} tokens in {dte:.1f} s on {threads} threads"})
    return out


# ------------------------------------------------------------ native ----

NOMINAL_HBM_GBS = 8000.0          # HBM3e nominal, for context beside the measured copy peak
SWEEP_B = (1, 8, 32, 128, 512)
SWEEP_C = (1, 2, 4, 8, 16)
SWEEP_STEPS = 512
EXTRA_WORKLOADS = ("kda-b128-h32-d128-c4", "kda-b128-h32-d128-c8",
                   "rwkv6-b128-h32-d64-c4", "rwkv6-b128-h32-d64-c8")


def working_set(w, R):
    bm = bytes_model(w)
    return R * w.heads * (bm["S"] + w.C * bm["E"])


def cold_layers(w, R, most=16):
    """Rotated layers for a workload's cold figures: at least R, and enough
    that the working set is at least 4x the L2 (at most `most`)."""
    r = R
    while working_set(w, r) < 4 * L2_BYTES and r < most:
        r += 1
    return r


def hot_cycle_us(w, args, dev, stream):
    """µs per layer-token of one layer's merge cycle decoded over and over,
    its whole working set resident in L2 (the hot figure beside the cold
    one; only for workloads whose layer fits in L2)."""
    from recurrent_state_head_b200 import binding as B
    rank = int(os.environ.get("RANK", "0"))
    su = Setup(w, 1, rank, dev)
    layers = su.layers(B.DL_MERGE_FOLD)
    outs = [L_.new_out(w.C) for L_ in layers]
    cyc = B.Cycle([L_.handle for L_ in layers], _ios(w, su.xs, outs, 1, w.C))
    ms = _time_graph(lambda: cyc.launch(stream), stream, args.steps, args.warmup, dev)
    ms, _ = reduce_over_ranks(ms / args.steps, 0, dev)
    cyc.close()
    return ms * 1e3 / w.C


def workload_config(w, R, world):
    """The `config` object of a bench line (the same keys in both arms)."""
    ws = working_set(w, R)
    l2 = (f"inputs larger than L2: {R} rotating layers, working set {ws / 1e6:.0f} MB vs L2 "
          f"{L2_BYTES / 1e6:.0f} MB" if ws >= L2_BYTES else
          f"working set {ws / 1e6:.1f} MB fits in L2 ({L2_BYTES / 1e6:.0f} MB): hot-cache figures")
    return {"workload": w.name, "op": ["gdn", "kda", "rwkv6"][w.op], "B": w.B, "H": w.H,
            "dk": w.dk, "dv": w.dv, "C": w.C, "layers_rotated": R,
            "inputs": f"q/k/v {w.in_dtype}, out {w.out_dtype}, fp32 state", "l2": l2,
            "step": f"one CUDA-graph merge cycle of {R} layers: {w.C - 1} appends + "
                    f"1 merge-token per layer, token-major",
            "parallelism": f"replicas{world}"}


class Setup:
    """States and C tokens of inputs of R independent layers (replica seeds)."""

    def __init__(self, w, R, rank, dev):
        from recurrent_state_head_b200 import device as D
        from recurrent_state_head_b200 import synth
        self.w, self.R, self.dev = w, R, dev
        ids = [rank * R + l for l in range(R)]
        self.S0 = [synth.initial_state(w, layer=i) for i in ids]
        self.bon = [synth.bonus(w, layer=i) for i in ids]
        self.xs = [D.to_device(synth.tokens(w, 0, w.C, layer=i, want64=False), w, dev) for i in ids]

    def layers(self, mode):
        from recurrent_state_head_b200 import device as D
        return [D.DecodeLayer(self.w, self.S0[l], self.bon[l], device=self.dev, auto_merge=mode)
                for l in range(self.R)]


def _ios(w, xs, outs, R, C):
    return [[(xs[l]["q"][t], xs[l]["k"][t], xs[l]["v"][t],
              None if w.op == 2 else xs[l]["beta"][t], xs[l]["g"][t], outs[l][t])
             for l in range(R)] for t in range(C)]


def _time_graph(launch, stream, steps, warmup, dev):
    import torch
    for _ in range(warmup):
        launch()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        launch()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1)


def kernel_durations(layers, xs, outs, w, R, C, stream, dev, reps, prime, merge_layers=None):
    """Per-launch device time of every kernel of a merge cycle, from CUDA
    timing events recorded on the launching stream between kernels.

    The kernels are launched through the C ABI with pointers prepared in
    advance, right after `prime()` (one cycle-graph launch) has queued a
    millisecond of GPU work, so that the host stays ahead of the GPU and the
    events bracket kernel time only.  These are isolated launches: inside
    the cycle graph consecutive kernels overlap their ramp and tail, so the
    sum of these durations exceeds the graph's step time.  layers: decode
    layers in merge-token mode (each dl_decode_step is one kernel);
    merge_layers (optional): layers with auto_merge off, for the separate
    merge kernel (dl_merge)."""
    import torch
    from recurrent_state_head_b200 import binding as B
    lib = B.lib()
    st = stream.cuda_stream

    def io(t, l):
        x = xs[l]
        return (x["q"][t].data_ptr(), x["k"][t].data_ptr(), x["v"][t].data_ptr(),
                None if w.op == 2 else x["beta"][t].data_ptr(), x["g"][t].data_ptr(),
                outs[l][t].data_ptr())

    ios = [[io(t, l) for l in range(R)] for t in range(C)]
    plan = []                                   # (kind, t, callable)
    for t in range(C):
        for l in range(R):
            h = layers[l].handle.h
            plan.append(("merge_token" if t == C - 1 else "append", t,
                         (lib.dl_decode_step, (h,) + ios[t][l] + (st,))))
    if merge_layers is not None:
        for t in range(C):
            for l in range(R):
                plan.append((None, t, (lib.dl_decode_step,
                                       (merge_layers[l].handle.h,) + ios[t][l] + (st,))))
        for l in range(R):
            plan.append(("merge", C, (lib.dl_merge, (merge_layers[l].handle.h, st))))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(plan) + 1)]
    out = {}
    for rep in range(reps + 1):
        prime()
        evs[0].record(stream)
        for i, (kind, t, (fn, args)) in enumerate(plan):
            rc = fn(*args)
            if rc != B.DL_OK:
                raise RuntimeError(f"launch failed: {B.dl_strerror(rc)}: {B.dl_last_error()}")
            evs[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        if rep == 0:
            continue                             # warm-up
        for i, (kind, t, _) in enumerate(plan):
            if kind is not None:
                out.setdefault((kind, t), []).append(evs[i].elapsed_time(evs[i + 1]))
    return out


def eager_graph(w, states, xs, outs, bons, R, C, stream, dev):
    """C tokens through R layers of the eager kernel, captured as one graph."""
    import torch
    from recurrent_state_head_b200 import binding as B
    from recurrent_state_head_b200 import device as D
    cfg = D.config_of(w)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for t in range(C):
                for l in range(R):
                    beta = None if w.op == 2 else xs[l]["beta"][t]
                    B.dl_eager_step(cfg, states[l], xs[l]["q"][t], xs[l]["k"][t], xs[l]["v"][t],
                                    beta, xs[l]["g"][t], bons[l], outs[l][t], side)
    stream.wait_stream(side)
    return g


def measure(w, R, args, dev, stream, peaks, headline):
    """Every figure of one workload: the graph-captured merge cycle (timed
    region), per-kernel durations, the separate-merge and staggered-slot
    cycles, the eager kernel.  Returns (result dict, objects kept for e2e)."""
    import torch
    from recurrent_state_head_b200 import binding as B

    rank = int(os.environ.get("RANK", "0"))
    C, NH = w.C, w.heads
    bm = bytes_model(w, fold=True)
    bm_sep = bytes_model(w, fold=False)
    su = Setup(w, R, rank, dev)
    xs = su.xs
    layers = su.layers(B.DL_MERGE_FOLD)
    outs = [L_.new_out(C) for L_ in layers]
    cycle = B.Cycle([L_.handle for L_ in layers], _ios(w, xs, outs, R, C))

    # --- timed region: K cycle launches
    for _ in range(args.warmup):
        cycle.launch(stream)
    torch.cuda.synchronize(dev)
    barrier(dev)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            cycle.launch(stream)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(dev)
    torch.cuda.synchronize(dev)
    tokens_local = w.B * C * R * args.steps          # decode tokens through one layer
    max_ms, tokens_all = reduce_over_ranks(ev0.elapsed_time(ev1), tokens_local, dev)
    ms_per_step = max_ms / args.steps
    us_per_token = ms_per_step * 1e3 / (C * R)
    gbs = NH * (bm["token_read"] + bm["token_write"]) * C * R / (ms_per_step / 1e3) / 1e9

    # --- per-kernel durations (isolated launches)
    merge_layers = su.layers(B.DL_MERGE_OFF)
    kd = kernel_durations(layers, xs, outs, w, R, C, stream, dev, reps=max(3, min(args.steps, 10)),
                          prime=lambda: cycle.launch(stream), merge_layers=merge_layers)
    del merge_layers
    app = {t: statistics.mean(kd[("append", t)]) for t in range(C - 1) if ("append", t) in kd}
    fold_us = statistics.mean(kd[("merge_token", C - 1)]) * 1e3 if ("merge_token", C - 1) in kd else None
    merge_us = statistics.mean(kd[("merge", C)]) * 1e3
    if app:
        app_avg_ms = statistics.mean(app.values())
        app_bytes = NH * statistics.mean([sum(bm["append"](L)) for L in app])
        dominant = "append_kernel"
    else:                                              # C = 1: every token is a merge-token
        app_avg_ms = fold_us / 1e3
        app_bytes = NH * sum(bm["merge_token"](0))
        dominant = "append_kernel (merge-token)"
    achieved = app_bytes / (app_avg_ms / 1e3) / 1e9
    res = {
        "value": tokens_all / (max_ms / 1e3), "ms_per_step": ms_per_step,
        "us_per_token": us_per_token, "hbm_gbs": gbs,
        "hbm_frac": gbs / peaks["hbm_gbs"], "hbm_frac_nominal": gbs / NOMINAL_HBM_GBS,
        "bytes_written_per_token": NH * bm["token_write"],
        "bytes_read_per_token": NH * bm["token_read"],
        "kernels": {"append_us_by_L": [app[L] * 1e3 for L in sorted(app)],
                    "append_avg_us": app_avg_ms * 1e3,
                    "merge_token_us": fold_us, "merge_us": merge_us,
                    "merge_gbs": NH * sum(bm["merge"](C)) / (merge_us / 1e6) / 1e9,
                    "timing": "isolated launches, CUDA events between kernels"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic(w.name), "kernel": dominant,
                     "peak_source": peaks["source"], "peak_nominal": NOMINAL_HBM_GBS,
                     "frac_nominal": achieved / NOMINAL_HBM_GBS,
                     "timing": "isolated launches of the kernel, mean over the cycle's log "
                               "lengths, CUDA events on the launching stream"},
        "gpu_launches": cycle.kernels * args.steps,
        "clocks": clk.summary(),
    }
    if fold_us:
        res["kernels"]["merge_token_gbs"] = NH * sum(bm["merge_token"](C - 1)) / (fold_us / 1e6) / 1e9
        res["kernels"]["merge_token_frac"] = res["kernels"]["merge_token_gbs"] / peaks["hbm_gbs"]

    # --- the same cycle with the merge as its own kernel (ablation)
    if args.ablation:
        sep = su.layers(B.DL_MERGE_SEPARATE)
        cyc_sep = B.Cycle([L_.handle for L_ in sep], _ios(w, xs, outs, R, C))
        ms = _time_graph(lambda: cyc_sep.launch(stream), stream, args.steps, args.warmup, dev)
        ms, _ = reduce_over_ranks(ms / args.steps, 0, dev)
        res["separate_merge"] = {
            "us_per_token": ms * 1e3 / (C * R),
            "hbm_gbs": NH * (bm_sep["token_read"] + bm_sep["token_write"]) * C * R / (ms / 1e3) / 1e9,
            "bytes_written_per_token": NH * bm_sep["token_write"]}
        cyc_sep.close()
        del sep

    # --- continuous batching: the slots at staggered log lengths (slot b
    #     joined b mod C tokens late), so every token of the cycle runs an
    #     append over 7/8 of the slots and a merge-token over the rest
    if args.staggered and C > 1:
        stag = su.layers(B.DL_MERGE_FOLD)
        for l, L_ in enumerate(stag):
            for t in range(C - 1):
                L_.step(xs[l], t, outs[l][t], stream=stream,
                        active=[(b % C) > t for b in range(w.B)])
        cyc_st = B.Cycle([L_.handle for L_ in stag], _ios(w, xs, outs, R, C))
        ms = _time_graph(lambda: cyc_st.launch(stream), stream, args.steps, args.warmup, dev)
        ms, _ = reduce_over_ranks(ms / args.steps, 0, dev)
        # each token of each layer is one slot-list launch: time them alone
        kd_st = kernel_durations(stag, xs, outs, w, R, C, stream, dev, reps=3,
                                 prime=lambda: cyc_st.launch(stream))
        slot_us = statistics.mean([x for v in kd_st.values() for x in v]) * 1e3
        res["staggered"] = {
            "us_per_token": ms * 1e3 / (C * R),
            "hbm_gbs": gbs * us_per_token / (ms * 1e3 / (C * R)),
            "kernels_per_step": cyc_st.kernels,
            "slot_kernel_us": slot_us,
            "slot_lengths": "slot b at b mod C when the cycle starts"}
        cyc_st.close()
        del stag

    # --- eager dense baseline, same layers and rotation, graph-captured
    if args.eager:
        eager_S = [L_.base.clone() for L_ in layers]
        g_eager = eager_graph(w, eager_S, xs, outs, [L_.bonus for L_ in layers], R, C, stream, dev)
        e_ms = _time_graph(g_eager.replay, stream, args.steps, args.warmup, dev) / args.steps
        e_ms, _ = reduce_over_ranks(e_ms, 0, dev)
        e_read, e_write = bm["eager"]
        res["eager"] = {
            "us_per_token": e_ms * 1e3 / (C * R),
            "tok_s": w.B * C * R * world_size() / (e_ms / 1e3),
            "hbm_gbs": NH * (e_read + e_write) * C * R / (e_ms / 1e3) / 1e9,
            "bytes_written_per_token": NH * e_write,
            "write_ratio_vs_deltalog": e_write / bm["token_write"],
            "speedup_deltalog": (e_ms * 1e3 / (C * R)) / us_per_token,
        }
        res["eager"]["hbm_frac"] = res["eager"]["hbm_gbs"] / peaks["hbm_gbs"]
        del g_eager, eager_S
    keep = {"setup": su, "layers": layers, "outs": outs, "cycle": cycle, "tokens_local": tokens_local}
    return res, keep


def world_size():
    return int(os.environ.get("WORLD_SIZE", "1"))


def e2e_overlapped(w, R, keep, args, dev, stream):
    """End to end through the public API with host buffers: every step
    copies that step's inputs from pinned host memory, launches the cycle
    (dl_cycle_launch) and copies the outputs back to pinned host memory.
    Each direction is one copy a step: the inputs of all layers sit in one
    pinned host buffer and one device buffer (the layers' q, k, v, beta, g
    are 256-byte aligned views into it), the outputs likewise.  Two device
    buffer sets alternate, with a cycle graph captured over each, so the
    inputs of step k+1 (one copy stream) and the outputs of step k-1
    (another) cross PCIe while step k computes; events order each buffer's
    reuse.  The timed region runs from before the first copy to after the
    last one, on the launching stream."""
    import torch
    from recurrent_state_head_b200 import binding as B
    names = ("q", "k", "v", "beta", "g")
    su, layers = keep["setup"], keep["layers"]
    C = w.C
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    pieces, off = [], 0                        # (layer, name, byte offset, tensor)
    for l in range(R):
        for n in names:
            t = su.xs[l][n]
            pieces.append((l, n, off, t))
            off += up(t.numel() * t.element_size())
    in_bytes = off
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for l, n, o, t in pieces:
        nb = t.numel() * t.element_size()
        host_in[o:o + nb].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
    o0 = layers[0].new_out(C)
    out_each = up(o0.numel() * o0.element_size())
    out_bytes = R * out_each
    sets = []
    for s_ in range(2):
        dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        xs_s = [{} for _ in range(R)]
        for l, n, o, t in pieces:
            nb = t.numel() * t.element_size()
            xs_s[l][n] = dev_in[o:o + nb].view(t.dtype).view(t.shape)
        dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        outs_s = [dev_out[l * out_each:l * out_each + o0.numel() * o0.element_size()].view(o0.dtype).view(o0.shape)
                  for l in range(R)]
        cyc = B.Cycle([L_.handle for L_ in layers], _ios(w, xs_s, outs_s, R, C))
        host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
        sets.append((dev_in, dev_out, cyc, host_out))
    h2d_bytes = sum(t.numel() * t.element_size() for _, _, _, t in pieces)
    d2h_bytes = R * o0.numel() * o0.element_size()
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ev_in, ev_done, ev_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def load(s_):
        with torch.cuda.stream(h2d):
            sets[s_][0].copy_(host_in, non_blocking=True)
            ev_in[s_].record(h2d)

    def run(K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d.wait_stream(stream)
        d2h.wait_stream(stream)
        load(0)
        for k in range(K):
            s_ = k % 2
            if k + 1 < K:
                s1 = (k + 1) % 2
                if k >= 1:
                    h2d.wait_event(ev_done[s1])       # step k-1 has read set s1
                load(s1)
            stream.wait_event(ev_in[s_])
            if k >= 2:
                stream.wait_event(ev_out[s_])         # step k-2's outputs are out
            sets[s_][2].launch(stream)
            ev_done[s_].record(stream)
            d2h.wait_event(ev_done[s_])
            with torch.cuda.stream(d2h):
                sets[s_][3].copy_(sets[s_][1], non_blocking=True)
                ev_out[s_].record(d2h)
        stream.wait_stream(d2h)
        stream.wait_stream(h2d)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    run(max(3, args.warmup))
    barrier(dev)
    e_ms = run(args.steps)
    barrier(dev)
    e_max, e_tok = reduce_over_ranks(e_ms, keep["tokens_local"], dev)
    for s_ in sets:
        s_[2].close()
    return {"value": e_tok / (e_max / 1e3), "unit": "tok/s",
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
            "ms_per_step": e_max / args.steps,
            "note": "pinned host inputs in, outputs out every step, one copy each way; two buffer "
                    "sets, copies on two copy streams overlapping the previous / next step's cycle"}


def run_sweep(args, dev, stream, peaks):
    """The 24-layer GDN stack (heads of the B128 H16 d128 workload), one
    decode step per layer in sequence, for every (B, C) cell: 512 steps per
    layer as 512 / C launches of one cycle graph over the stack.  Stacks
    smaller than 4x L2 are replicated and the replicas decoded in turn, so
    that every base read comes from HBM (hot figures, one stack, alongside).
    States and inputs are drawn on the device (torch's generator, the
    workloads' distributions): 12 GB of state at B = 512 is too much to
    draw on the host in a benchmark."""
    import torch
    from recurrent_state_head_b200 import binding as B
    from recurrent_state_head_b200 import device as D
    from recurrent_state_head_b200 import synth

    rank = int(os.environ.get("RANK", "0"))
    gen = torch.Generator(device=dev)
    gen.manual_seed(4_000 + rank)
    cells = []
    steps, warm = SWEEP_STEPS, max(3, args.warmup)
    with ClockSampler(dev) as clk:
        for Bsz in SWEEP_B:
            w16 = synth.WORKLOADS[f"gdn-stack24-b{Bsz}-h16-d128-c16"]
            NH, nl = w16.heads, w16.layers
            stack_state = nl * NH * 4 * w16.dk * w16.dv
            reps = max(1, math.ceil(4 * L2_BYTES / stack_state))
            R = nl * reps
            bases = [D.draw_state(w16, l, dev, gen) for l in range(R)]
            xs = [D.draw_tokens(w16, max(SWEEP_C), dev, gen) for l in range(R)]
            outs = [torch.empty((max(SWEEP_C), NH, w16.dv), dtype=torch.bfloat16, device=dev)
                    for _ in range(R)]
            for C in SWEEP_C:
                w = synth.WORKLOADS[f"gdn-stack24-b{Bsz}-h16-d128-c{C}"]
                bm = bytes_model(w)
                layers = [D.DecodeLayer(w, bases[l], None, device=dev) for l in range(R)]
                cyc = B.Cycle([L_.handle for L_ in layers], _ios(w, xs, outs, R, C))
                n = steps // C
                ms = _time_graph(lambda: cyc.launch(stream), stream, n, warm, dev)
                ms, _ = reduce_over_ranks(ms, 0, dev)
                us = ms * 1e3 / (n * C * R)
                cell = {"B": Bsz, "C": C, "state_MB_per_stack": stack_state / 2 ** 20,
                        "replicas": reps, "deltalog_us_per_token": us,
                        "deltalog_gbs": NH * (bm["token_read"] + bm["token_write"]) / us / 1e3,
                        "deltalog_write_bytes_per_token": NH * bm["token_write"],
                        "kernels_per_launch": cyc.kernels}
                cell["deltalog_hbm_frac"] = cell["deltalog_gbs"] / peaks["hbm_gbs"]
                if reps > 1:
                    hot = B.Cycle([L_.handle for L_ in layers[:nl]], _ios(w, xs, outs, nl, C))
                    hms = _time_graph(lambda: hot.launch(stream), stream, n, warm, dev)
                    hms, _ = reduce_over_ranks(hms, 0, dev)
                    cell["deltalog_us_per_token_hot"] = hms * 1e3 / (n * C * nl)
                    hot.close()
                cyc.close()
                del layers
                g = eager_graph(w, bases, xs, outs, [None] * R, R, C, stream, dev)
                ems = _time_graph(g.replay, stream, n, warm, dev)
                ems, _ = reduce_over_ranks(ems, 0, dev)
                e_read, e_write = bm["eager"]
                eus = ems * 1e3 / (n * C * R)
                cell.update({"eager_us_per_token": eus,
                             "eager_gbs": NH * (e_read + e_write) / eus / 1e3,
                             "eager_write_bytes_per_token": NH * e_write,
                             "speedup": eus / us, "write_ratio": e_write / bm["token_write"]})
                del g
                cells.append(cell)
            del bases, xs, outs
            torch.cuda.empty_cache()
    return {"steps": steps, "layers": 24, "cells": cells, "clocks": clk.summary(),
            "unit": "µs per layer-token (amortised over the cycle)",
            "inputs": "device-drawn (torch Philox), workload distributions; C tokens of inputs "
                      "reused every launch"}


def run_native(args, rank, world, local_rank):
    import torch
    from recurrent_state_head_b200 import binding as B
    from recurrent_state_head_b200 import synth

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    B.lib()                                   # fail loudly if the library is missing

    w = synth.WORKLOADS[args.workload]
    R = args.layers
    stream = torch.cuda.current_stream(dev)
    peaks = measured_peaks()
    res, keep = measure(w, R, args, dev, stream, peaks, headline=True)
    result = {
        "metric": METRIC, "value": res.pop("value"), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "config": workload_config(w, R, world),
    }
    result.update(res)
    if args.e2e:
        result["e2e"] = e2e_overlapped(w, R, keep, args, dev, stream)
    keep["cycle"].close()
    del keep
    torch.cuda.empty_cache()

    # --- the other operators at one GPU (GDN, KDA, RWKV6 at C = 4 and 8)
    if args.workloads:
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            wx = synth.WORKLOADS[name]
            Rw = cold_layers(wx, R)
            r, k = measure(wx, Rw, args, dev, stream, peaks, headline=False)
            k["cycle"].close()
            del k
            torch.cuda.empty_cache()
            extra[name] = {
                "us_per_token": r["us_per_token"], "tok_s": r["value"], "hbm_gbs": r["hbm_gbs"],
                "hbm_frac": r["hbm_frac"], "hbm_frac_nominal": r["hbm_frac_nominal"],
                "append_avg_us": r["kernels"]["append_avg_us"],
                "append_roofline_frac": r["roofline"]["frac"],
                "merge_token_us": r["kernels"]["merge_token_us"],
                "merge_token_frac": r["kernels"].get("merge_token_frac"),
                "merge_us": r["kernels"]["merge_us"],
                "bytes_written_per_token": r["bytes_written_per_token"],
                "clocks": r["clocks"], "config": workload_config(wx, Rw, world),
            }
            if working_set(wx, 1) < L2_BYTES:
                extra[name]["hot_us_per_token"] = hot_cycle_us(wx, args, dev, stream)
                torch.cuda.empty_cache()
            if "eager" in r:
                extra[name].update({"eager_us_per_token": r["eager"]["us_per_token"],
                                    "eager_hbm_frac": r["eager"]["hbm_frac"],
                                    "write_ratio": r["eager"]["write_ratio_vs_deltalog"],
                                    "speedup": r["eager"]["speedup_deltalog"]})
            if "separate_merge" in r:
                extra[name]["separate_merge_us_per_token"] = r["separate_merge"]["us_per_token"]
            if "staggered" in r:
                extra[name]["staggered_us_per_token"] = r["staggered"]["us_per_token"]
        result["workloads"] = extra

    # --- the 24-layer stack: state-size and interval sweep
    if args.sweep:
        result["sweep"] = run_sweep(args, dev, stream, peaks)

    if rank == 0 and world == 1 and args.cpu_baseline:
        result["cpu_baseline"] = cpu_oracle_sample(w)
    return result


# ---------------------------------------------------------- reference ---

def run_reference(args, rank, world):
    """The oracle as the reference arm: host cores, bounded samples."""
    from recurrent_state_head_b200 import synth
    if rank != 0:
        return None
    w = synth.WORKLOADS[args.workload]
    per_step_s = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, target_s=per_step_s, extras=False)
    vals, samples = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_oracle_sample(w, target_s=per_step_s, extras=False)
        vals.append(r["value"])
        samples.append(r)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    ms_per_step = wall * 1e3 / max(1, args.steps)
    last = samples[-1]
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.layers, world),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--no-eager", dest="eager", action="store_false")
    ap.add_argument("--no-staggered", dest="staggered", action="store_false",
                    help="skip the cycle with slots at staggered log lengths")
    ap.add_argument("--no-ablation", dest="ablation", action="store_false",
                    help="skip the separate-merge cycle")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-workloads", dest="workloads", action="store_false",
                    help="skip the KDA and RWKV6 workloads")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false",
                    help="skip the 24-layer stack sweep")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_native(args, rank, world, local_rank)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    try:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
