#!/usr/bin/env python
"""Throughput of the B200 SSD scan (and decode step) on synthetic workloads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--also A,B] [--impl ours|reference]

The headline line is the largest single-GPU scan workload (c3_long: one
65536-token row, 80 heads in 8 groups, carried initial state); the other scan
workloads (c1_130m, c2_2p7b) are timed in the same run and nested under
"configs" with the same keys, the decode step under "decode" and the
backward under "backward".

A "step" is one chunked forward scan (every stage of the hot path: dt
preparation, chunk cumsum, intra-chunk C.B^T, chunk states, state passing,
chunk output) over one batch of the workload; the decode workload's step is
one single-token state update.  The K timed steps are captured once into a
CUDA graph and launched as one graph, so the number is device time, not
Python call overhead; per-kernel times come from an eager traced pass.  Rank 0 prints ONE JSON line.  With N > 1 each
rank runs its own copy of the workload (independent batches, no collective on
the data path: weak scaling); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method
has) on a bounded sample of the same workload, on this host's cores.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from state_space_sequence_scan_b200.inputs import (  # noqa: E402
    SCAN_CONFIGS, STEP_CONFIGS, make_scan_inputs, make_step_inputs)

L2_BYTES = 126 * 1024 * 1024
METRIC = "SSD chunked-scan Mtokens/s & % roofline; decode state-update HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------
# algorithmic work (bytes every implementation must move, flops of the causal
# chunked form with C.B^T counted once per group)

def states_bytes(cfg) -> float:
    """The chunk-boundary states [b, nc, H, N, P] fp32 (--chunk-states)."""
    nc = math.ceil(cfg.seqlen / cfg.chunk_size)
    return float(cfg.batch * nc * cfg.nheads * cfg.state_dim * cfg.head_dim * 4)


def scan_bytes(cfg, states=False) -> float:
    b, L, H, P, N, G = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    e = 4 if cfg.dtype == "f32" else 2
    tok = b * L
    byt = tok * H * P * e + 2 * tok * G * N * e + tok * H * 4   # x, B, C, dt_raw
    byt += tok * H * P * 4                                      # y (fp32)
    byt += b * H * N * P * 4 * (2 if cfg.init == "normal" else 1)  # init (if any) + final state
    byt += 3 * H * 4
    return float(byt) + (states_bytes(cfg) if states else 0.0)


def scan_flops(cfg) -> float:
    b, L, H, P, N, G, Q = (cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups,
                           cfg.chunk_size)
    nc = math.ceil(L / Q)
    per_chunk = G * Q * (Q + 1) * N + H * (Q * (Q + 1) * P + 4 * Q * N * P)
    return float(b * nc * per_chunk)


def step_bytes(cfg) -> float:
    b, H, P, N, G = cfg.batch, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    e = 4 if cfg.dtype == "f32" else 2
    return float(2 * b * H * N * P * 4 + b * H * P * e + 2 * b * G * N * e + b * H * 4 + b * H * P * 4 + 3 * H * 4)


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the
# dominant kernel, from one ncu capture each.  Each entry names the source file
# of the kernel and the first 16 hex digits of its sha256 at capture time: once
# that file changes the number no longer describes the kernel and the bench
# reports null.
NCU_TRAFFIC = {
    ("c3_long", "tc_chunk_out"): (2314.120448e6, "state_space_sequence_scan_b200/csrc/ssd_scan_tc.cu",
                                  "6e213af5e95844a6"),
    ("c2_2p7b", "tc_chunk_out"): (1017.629440e6, "state_space_sequence_scan_b200/csrc/ssd_scan_tc.cu",
                                  "6e213af5e95844a6"),
    ("c4_decode", "decode_step"): (1291.7568e6, "state_space_sequence_scan_b200/csrc/ssd_step.cu",
                                   "a5f3c2cec738b994"),
}


def measured_traffic(workload, kernel):
    """(bytes per launch, description) if the capture still describes the kernel, else (None, None)."""
    import hashlib
    e = NCU_TRAFFIC.get((workload, kernel))
    if e is None:
        return None, None
    nbytes, src, digest = e
    try:
        with open(os.path.join(ROOT, src), "rb") as f:
            cur = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None, None
    if cur != digest:
        return None, None
    return nbytes, "ncu capture of %s on %s (source sha256 %s)" % (kernel, workload, digest)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------------------

def init_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, ws: int) -> float:
    if ws == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _dev_sets(inp, nsets, device):
    """nsets device copies of the inputs (rotated so timed steps never hit L2)."""
    sets = []
    for _ in range(nsets):
        sets.append({k: (v.to(device) if v is not None else None) for k, v in inp.items()})
    return sets


def bench_scan(cfg, args, ws, rank, local):
    from state_space_sequence_scan_b200 import ssd
    dev = torch.device("cuda", local)
    inp = make_scan_inputs(cfg, seed=cfg.seed + 1000 * rank)
    one = scan_bytes(cfg, args.chunk_states)
    nsets = max(1, min(8, math.ceil(3 * L2_BYTES / one)))
    sets = _dev_sets(inp, nsets, dev)
    b, L, H, P, N, G, Q = (cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups,
                           cfg.chunk_size)
    nc = math.ceil(L / Q)
    outs = [(torch.empty(b, L, H, P, device=dev), torch.empty(b, H, N, P, device=dev),
             torch.empty(b, nc, H, N, P, device=dev) if args.chunk_states else None) for _ in range(nsets)]
    wsz = ssd.workspace_size(b, L, H, P, N, G, Q, sets[0]["x"].dtype, args.path)
    work = ssd.alloc_workspace(wsz, dev)
    seqs = None
    if args.packed:
        # documents of about 512 tokens (seeded lengths), the same ids for every set
        import numpy as np
        rng = np.random.default_rng(cfg.seed + 5)
        ids = np.zeros((b, L), np.int32)
        for bi in range(b):
            cuts = np.sort(rng.integers(1, L, size=max(1, L // 512)))
            ids[bi] = np.searchsorted(cuts, np.arange(L), side="right")
        seqs = torch.from_numpy(ids).to(dev)

    def step(k):
        s = sets[k % nsets]
        y, fs, cs = outs[k % nsets]
        if seqs is not None:
            ssd.chunk_scan_fwd_varlen(s["x"], s["dt_raw"], s["dt_bias"], s["A"], s["B"], s["C"], s["D"], seqs,
                                      init_state=s["init_state"], chunk_size=Q, path=args.path, workspace=work)
        elif cs is None:
            ssd.chunk_scan_fwd(s["x"], s["dt_raw"], s["dt_bias"], s["A"], s["B"], s["C"], s["D"],
                               init_state=s["init_state"], chunk_size=Q, path=args.path, workspace=work, y=y,
                               final_state=fs)
        else:
            ssd.chunk_scan_fwd_states(s["x"], s["dt_raw"], s["dt_bias"], s["A"], s["B"], s["C"], s["D"],
                                      init_state=s["init_state"], chunk_size=Q, path=args.path, workspace=work,
                                      y=y, final_state=fs, chunk_states=cs)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    if ssd.read_device_status(work) != 0:
        raise RuntimeError("device status %d after warm-up" % ssd.read_device_status(work))

    graph = capture_steps(step, args.steps)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()                     # exactly K steps, launched as one CUDA graph
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, ws)
    del graph

    # per-kernel device times: the same K steps again, eagerly, with event brackets
    ssd.trace_enable(min(8192, 8 * args.steps + 8))
    for k in range(args.steps):
        step(k)
    torch.cuda.synchronize()
    trace = ssd.trace_read()
    ssd.trace_enable(0)
    launches_per_step = sum(n for n, _ in trace.values()) / max(args.steps, 1)

    res = dict(ms=ms_max, tokens=cfg.tokens, bytes=one, flops=scan_flops(cfg), clocks=clk, trace=trace,
               launches=int(round(launches_per_step * args.steps)), nsets=nsets)
    res["e2e"] = e2e_scan(inp, cfg, args, dev, work)
    return res


def capture_steps(step, steps):
    """A CUDA graph holding exactly `steps` calls of step(k): the timed
    region then costs one launch instead of `steps` Python/ctypes calls."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for k in range(steps):
            step(k)
    torch.cuda.synchronize()
    return g


def e2e_scan(inp, cfg, args, dev, work):
    """Same metric through the public call with host buffers: every step
    copies its inputs in from pinned host memory, runs the scan and copies y
    and final_state (and with --chunk-states the chunk-boundary states) back.
    Steps are pipelined the way a caller streaming batches would run them:
    two device and two pinned host buffer sets, the copies in on one stream,
    the scans on another, the copies out on a third, so that step k+1's
    inputs cross PCIe while step k computes and step k-1's results come back
    (the link is full duplex).  Timed with CUDA events from the first copy in
    to the last copy out."""
    from state_space_sequence_scan_b200 import ssd
    b, L, H, P, N, Q = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.chunk_size
    nc = math.ceil(L / Q)
    host = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
    slots = []
    for _ in range(2):
        sl = {"d": {k: (torch.empty_like(v, device=dev) if v is not None else None) for k, v in inp.items()},
              "y": torch.empty(b, L, H, P, device=dev), "fs": torch.empty(b, H, N, P, device=dev),
              "y_h": torch.empty(b, L, H, P).pin_memory(), "fs_h": torch.empty(b, H, N, P).pin_memory(),
              "cs": torch.empty(b, nc, H, N, P, device=dev) if args.chunk_states else None,
              "cs_h": torch.empty(b, nc, H, N, P).pin_memory() if args.chunk_states else None}
        slots.append(sl)
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = (slots[0]["y_h"].numel() * 4 + slots[0]["fs_h"].numel() * 4 +
           (slots[0]["cs_h"].numel() * 4 if args.chunk_states else 0))
    steps = max(3, min(args.steps, 20))
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("in", "cmp", "out")}

    def one(k):
        sl = slots[k % 2]
        e_in, e_cmp, e_out = ev["in"][k % 2], ev["cmp"][k % 2], ev["out"][k % 2]
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(e_out)          # step k-2 is done with this slot (its scan and its copy out)
            for kk, v in host.items():
                if v is not None:
                    sl["d"][kk].copy_(v, non_blocking=True)
            e_in.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(e_in)
            d = sl["d"]
            if sl["cs"] is None:
                ssd.chunk_scan_fwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                   init_state=d["init_state"], chunk_size=Q, path=args.path, workspace=work,
                                   y=sl["y"], final_state=sl["fs"])
            else:
                ssd.chunk_scan_fwd_states(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                          init_state=d["init_state"], chunk_size=Q, path=args.path,
                                          workspace=work, y=sl["y"], final_state=sl["fs"], chunk_states=sl["cs"])
            e_cmp.record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_cmp)
            sl["y_h"].copy_(sl["y"], non_blocking=True)
            sl["fs_h"].copy_(sl["fs"], non_blocking=True)
            if sl["cs"] is not None:
                sl["cs_h"].copy_(sl["cs"], non_blocking=True)
            e_out.record(s_out)

    for k in range(2):
        one(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(steps):
        one(k)
    s_out.synchronize()
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    if ssd.read_device_status(work) != 0:
        raise RuntimeError("device status %d after the end-to-end steps" % ssd.read_device_status(work))
    return dict(ms_per_step=ms, h2d=h2d, d2h=d2h, steps=steps, pipelined="2 buffer sets, 3 streams")


def bench_step(cfg, args, ws, rank, local):
    from state_space_sequence_scan_b200 import ssd
    dev = torch.device("cuda", local)
    ntok = 32
    inp = make_step_inputs(cfg, steps=ntok, seed=cfg.seed + 1000 * rank)
    d = {k: v.to(dev) for k, v in inp.items()}
    state = d["state"].clone()
    b, H, P = cfg.batch, cfg.nheads, cfg.head_dim
    y = torch.empty(b, H, P, device=dev)

    def step(k):
        t = k % ntok
        ssd.step(d["x"][t], d["dt_raw"][t], d["dt_bias"], d["A"], d["B"][t], d["C"][t], d["D"], state, y=y)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    graph = capture_steps(step, args.steps)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    ms_max = max_over_ranks(e0.elapsed_time(e1), ws)
    del graph
    ssd.trace_enable(min(8192, args.steps + 8))
    for k in range(args.steps):
        step(k)
    torch.cuda.synchronize()
    trace = ssd.trace_read()
    ssd.trace_enable(0)

    # e2e: pinned host token inputs in, y out, state resident (it is the cache)
    host = {k: inp[k][0].contiguous().pin_memory() for k in ("x", "dt_raw", "B", "C")}
    dd = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    y_h = torch.empty(b, H, P).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y_h.numel() * 4
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n2 = max(3, min(args.steps, 50))
    f0.record()
    for _ in range(n2):
        for k, v in host.items():
            dd[k].copy_(v, non_blocking=True)
        ssd.step(dd["x"], dd["dt_raw"], d["dt_bias"], d["A"], dd["B"], dd["C"], d["D"], state, y=y)
        y_h.copy_(y, non_blocking=True)
    f1.record()
    torch.cuda.synchronize()
    e2e = dict(ms_per_step=f0.elapsed_time(f1) / n2, h2d=h2d, d2h=d2h, steps=n2)
    return dict(ms=ms_max, bytes=step_bytes(cfg), clocks=clk, trace=trace,
                launches=sum(n for n, _ in trace.values()), e2e=e2e)


def dominant(trace):
    if not trace:
        return None, 0, 0.0
    name = max(trace, key=lambda k: trace[k][1])
    n, ms = trace[name]
    return name, n, ms


# algorithmic bytes each traced kernel must move (per launch), as fractions of the call
def bench_stage(cfg, args, local, peaks, peak_kind):
    """--stage conv1d | gated_norm: one of the steps either side of the scan,
    alone, on the workload's shapes (conv: x|B|C channels of width 4 from
    bf16 inputs; norm: y f32 and z bf16 over groups of H*P/G channels).  HBM
    bytes: conv reads xbc and writes x, B, C; the norm reads y and z and
    writes out (weights are negligible).  Timed like the scan: inputs rotated
    past L2, K steps in one CUDA graph, CUDA events on the launching stream."""
    from state_space_sequence_scan_b200 import ssd
    dev = torch.device("cuda", local)
    b, L, H, P, N, G = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    gen = torch.Generator().manual_seed(cfg.seed + 77)
    if args.stage == "conv1d":
        Cd, K = H * P + 2 * G * N, 4
        one = 2.0 * b * L * Cd * 2
        nsets = max(1, min(8, math.ceil(3 * L2_BYTES / one)))
        w = (torch.randn(Cd, K, generator=gen) / 2).to(dev)
        bias = (0.1 * torch.randn(Cd, generator=gen)).to(dev)
        sets = [torch.randn(b, L, Cd, generator=gen).to(torch.bfloat16).to(dev) for _ in range(nsets)]
        outs = [(torch.empty(b, L, H, P, dtype=torch.bfloat16, device=dev),
                 torch.empty(b, L, G, N, dtype=torch.bfloat16, device=dev),
                 torch.empty(b, L, G, N, dtype=torch.bfloat16, device=dev)) for _ in range(nsets)]
        lib = ssd.load_library()

        def step(k):
            x, B, C = outs[k % nsets]
            st = lib.ssd_conv1d_silu_split(sets[k % nsets].data_ptr(), w.data_ptr(), bias.data_ptr(), x.data_ptr(),
                                           B.data_ptr(), C.data_ptr(), b, L, H, P, G, N, K, 1,
                                           torch.cuda.current_stream(dev).cuda_stream)
            if st != 0:
                raise RuntimeError("ssd_conv1d_silu_split: %d" % st)
        kname = "conv1d_silu"
    else:
        D, grp = H * P, H * P // G
        one = float(b * L * D * (4 + 2 + 4))
        nsets = max(1, min(8, math.ceil(3 * L2_BYTES / one)))
        wt = (torch.rand(D, generator=gen) + 0.5).to(dev)
        sets = [(torch.randn(b * L, D, generator=gen).to(dev),
                 torch.randn(b * L, D, generator=gen).to(torch.bfloat16).to(dev)) for _ in range(nsets)]
        outs = [torch.empty(b * L, D, device=dev) for _ in range(nsets)]
        lib = ssd.load_library()

        def step(k):
            y, z = sets[k % nsets]
            st = lib.ssd_gated_rmsnorm(y.data_ptr(), z.data_ptr(), wt.data_ptr(), outs[k % nsets].data_ptr(), b * L, D,
                                       grp, 1e-5, 1, torch.cuda.current_stream(dev).cuda_stream)
            if st != 0:
                raise RuntimeError("ssd_gated_rmsnorm: %d" % st)
        kname = "gated_rmsnorm"
    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    graph = capture_steps(step, args.steps)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = one / (ms * 1e-3) / 1e9
    return {"stage": args.stage, "metric": "%s HBM GB/s" % args.stage, "value": gbs, "unit": "GB/s",
            "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup, "dtype": "bf16-in",
            "config": {"workload": cfg.name, "batch": b, "seqlen": L, "heads": H, "head_dim": P, "groups": G,
                       "state_dim": N, "l2": "rotating %d sets" % nsets},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / hbm, "kernel_bytes": one, "traffic": None,
                         "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind},
            "clocks": clk}


def bench_conv_scan(cfg, args, local, peaks, peak_kind):
    """--stage conv_scan (and nested in the default scan line): the conv1d
    (width 4, bf16) and the scan in the two arrangements on the workload's
    shapes.  split: ssd_conv1d_silu_split writes x, B, C, then
    ssd_chunk_scan_fwd reads them; combined: ssd_conv_scan_fwd reads xbc and
    convolves inside the scan's kernels.  Same inputs, K steps of each in one
    CUDA graph, inputs rotated past L2.  Bytes are the algorithmic HBM bytes
    of each arrangement: the split one also writes and reads x, B and C."""
    from state_space_sequence_scan_b200 import ssd
    dev = torch.device("cuda", local)
    b, L, H, P, N, G = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    Q = cfg.chunk_size
    Cd = H * P + 2 * G * N
    xbc_bytes = 2.0 * b * L * Cd
    scan_b = scan_bytes(cfg)
    split_bytes = 2 * xbc_bytes + scan_b                 # conv reads xbc, writes x|B|C; the scan reads them
    comb_bytes = scan_b                                  # xbc in place of x, B, C (the same bytes)
    nsets = max(1, min(8, math.ceil(3 * L2_BYTES / split_bytes)))
    gen = torch.Generator().manual_seed(cfg.seed + 91)
    inp = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in make_scan_inputs(cfg).items()}
    w = (torch.randn(Cd, 4, generator=gen) / 2).to(dev)
    bias = (0.1 * torch.randn(Cd, generator=gen)).to(dev)
    sets = [torch.randn(b, L, Cd, generator=gen).to(torch.bfloat16).to(dev) for _ in range(nsets)]
    xs = [(torch.empty(b, L, H, P, dtype=torch.bfloat16, device=dev),
           torch.empty(b, L, G, N, dtype=torch.bfloat16, device=dev),
           torch.empty(b, L, G, N, dtype=torch.bfloat16, device=dev)) for _ in range(nsets)]
    ys = [torch.empty(b, L, H, P, device=dev) for _ in range(nsets)]
    fs = torch.empty(b, H, N, P, device=dev)
    wsz = ssd.workspace_size(b, L, H, P, N, G, Q, torch.bfloat16, "tensor")
    wsp = ssd.alloc_workspace(wsz, dev)
    lib = ssd.load_library()
    stream = torch.cuda.current_stream(dev)

    def split(k):
        x, B, C = xs[k % nsets]
        # the stream current at call time: under graph capture, the capturing one
        st = lib.ssd_conv1d_silu_split(sets[k % nsets].data_ptr(), w.data_ptr(), bias.data_ptr(), x.data_ptr(),
                                       B.data_ptr(), C.data_ptr(), b, L, H, P, G, N, 4, 1,
                                       torch.cuda.current_stream(dev).cuda_stream)
        if st != 0:
            raise RuntimeError("ssd_conv1d_silu_split: %d" % st)
        ssd.chunk_scan_fwd(x, inp["dt_raw"], inp["dt_bias"], inp["A"], B, C, inp["D"], init_state=inp["init_state"],
                           chunk_size=Q, path="tensor", workspace=wsp, y=ys[k % nsets], final_state=fs)

    def combined(k):
        ssd.conv_scan_fwd(sets[k % nsets], w, bias, inp["dt_raw"], inp["dt_bias"], inp["A"], inp["D"], H, P, G, N,
                          init_state=inp["init_state"], chunk_size=Q, workspace=wsp, y=ys[k % nsets],
                          final_state=fs)

    res = {}
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for nm, fn in (("split", split), ("combined", combined)):
        for k in range(args.warmup):
            fn(k)
        torch.cuda.synchronize()
        graph = capture_steps(fn, args.steps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        byt = split_bytes if nm == "split" else comb_bytes
        res[nm] = {"ms_per_step": ms, "mtokens_per_s": b * L / (ms * 1e-3) / 1e6, "hbm_bytes": byt,
                   "hbm_gbs": byt / (ms * 1e-3) / 1e9}
        del graph
    clk = clocks.stop()
    if ssd.read_device_status(wsp) != 0 or ssd.read_device_status(None) != 0:
        raise RuntimeError("conv_scan: device status not ok")
    return {"stage": "conv_scan", "metric": "conv1d + scan Mtokens/s (combined arrangement)",
            "value": res["combined"]["mtokens_per_s"], "unit": "Mtokens/s", "higher_is_better": True,
            "steps": args.steps, "warmup": args.warmup, "dtype": "bf16-in/f32",
            "config": {"workload": cfg.name, "batch": b, "seqlen": L, "heads": H, "head_dim": P, "groups": G,
                       "state_dim": N, "chunk_size": Q, "conv_width": 4, "l2": "rotating %d sets" % nsets},
            "arrangements": res, "bytes_saved": split_bytes - comb_bytes,
            "speedup_combined_over_split": res["split"]["ms_per_step"] / res["combined"]["ms_per_step"],
            "clocks": clk}


# fp32 FMA throughput of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 flop x
# 1965 MHz (the clocks.max.sm of these B200s) = 74.45 TFLOP/s.
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1965e6 / 1e12


def bwd_flops(cfg):
    """Algorithmic FLOPs of the backward per call, causal triangles counted
    once: (whole call, the bwd_cols kernel's share).  Per (batch, chunk of q
    tokens): C.B^T once per group, G q(q+1) N; per head the dy.x^T pairs and
    the dx pairs, 2 q(q+1) P; the dB and dC pairs, 2 q(q+1) N; and ten
    q N P products (the forward's chunk state, the reverse pass's, the G_c
    terms of dx and dB, the H_in term of dC)."""
    b, L, H, P, N, G, Q = (cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups,
                           cfg.chunk_size)
    tot = cols = 0.0
    for c in range((L + Q - 1) // Q):
        q = min(Q, L - c * Q)
        T = q * (q + 1)
        tot += G * T * N + H * (2 * T * P + 2 * T * N + 10 * q * N * P)
        cols += G * T * N + H * (2 * T * P + T * N + 4 * q * N * P)
    return b * tot, b * cols


def bench_backward(cfg, args, local, peaks, peak_kind):
    """--stage backward: the deterministic backward (ssd_chunk_scan_bwd) on
    the workload's shapes, inputs and upstream gradients rotated past L2, K
    calls in one CUDA graph, CUDA events on the launching stream; then the
    same K calls eagerly with the library's per-kernel event brackets for
    the kernel shares.  bf16 layers with P 64, N 128 and Q a multiple of 128
    take the tensor-core pair kernels (roofline: the dense bf16/fp16 tensor
    peak), and the fp32 CUDA-core path is timed beside them under "simt";
    other layers take the CUDA-core path (roofline: the fp32 ALU peak,
    FP32_ALU_TFLOPS).  The HBM time of the algorithmic bytes is reported
    beside it."""
    from state_space_sequence_scan_b200 import ssd
    from state_space_sequence_scan_b200.inputs import make_grad_inputs
    dev = torch.device("cuda", local)
    b, L, H, P, N, G, Q = (cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups,
                           cfg.chunk_size)
    e = 4 if cfg.dtype == "f32" else 2
    tok, st = b * L, b * H * N * P * 4
    nbytes = float(tok * (H * P * e + 2 * G * N * e + H * 4)          # x, B, C, dt_raw
                   + tok * H * P * 4 + st * (2 if cfg.init == "normal" else 1)   # dy, dfinal, init
                   + tok * (H * P * 4 + H * 4 + 2 * G * N * 4) + st)   # dx, ddt_raw, dB, dC, dinit
    nsets = max(1, min(4, math.ceil(3 * L2_BYTES / nbytes)))
    sets, outs = [], []
    for k in range(nsets):
        inp = make_scan_inputs(cfg, seed=cfg.seed + 31 * k)
        gr = make_grad_inputs(cfg, seed=cfg.seed + 31 * k)
        sets.append(({kk: (v.to(dev) if v is not None else None) for kk, v in inp.items()},
                     gr["dy"].to(dev), gr["dfinal"].to(dev)))
        outs.append({"x": torch.empty(b, L, H, P, device=dev), "dt_raw": torch.empty(b, L, H, device=dev),
                     "dt_bias": torch.empty(H, device=dev), "A": torch.empty(H, device=dev),
                     "B": torch.empty(b, L, G, N, device=dev), "C": torch.empty(b, L, G, N, device=dev),
                     "D": torch.empty(H, device=dev), "init_state": torch.empty(b, H, N, P, device=dev)})
    work = ssd.alloc_workspace(ssd.bwd_workspace_size(b, L, H, P, N, G, Q, sets[0][0]["x"].dtype), dev)

    def timed(path):
        def step(k):
            d, dy, df = sets[k % nsets]
            ssd.chunk_scan_bwd(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"], dy,
                               dfinal_state=df, init_state=d["init_state"], chunk_size=Q, workspace=work,
                               out=outs[k % nsets], path=path)

        for k in range(args.warmup):
            step(k)
        torch.cuda.synchronize()
        if ssd.read_device_status(work) != 0:
            raise RuntimeError("device status %d after warm-up" % ssd.read_device_status(work))
        graph = capture_steps(step, args.steps)
        stream = torch.cuda.current_stream(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(local)
        clocks.start()
        time.sleep(0.3)
        torch.cuda.synchronize()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        ms = e0.elapsed_time(e1) / args.steps
        del graph
        ssd.trace_enable(min(8192, 16 * args.steps + 16))
        for k in range(args.steps):
            step(k)
        torch.cuda.synchronize()
        trace = ssd.trace_read()
        ssd.trace_enable(0)
        if ssd.read_device_status(work) != 0:
            raise RuntimeError("device status %d after the %s backward" % (ssd.read_device_status(work), path))
        return ms, trace, clk

    # the tensor-core pair kernels where they apply (bf16, P 64, N 128, Q a multiple of 128), else SIMT
    tensor = cfg.dtype == "bf16" and P == 64 and N == 128 and Q % 128 == 0
    path = "tensor" if tensor else "simt"
    ms, trace, clk = timed(path)
    simt = None
    if tensor:
        sms, strace, _ = timed("simt")
        simt = {"ms_per_step": sms, "mtokens_per_s": tok / (sms * 1e-3) / 1e6,
                "shares": {k: round(v[1] / max(sum(x[1] for x in strace.values()), 1e-12), 4)
                           for k, v in strace.items()}}
    tot_ms = sum(v[1] for v in trace.values())
    flops, cols_flops = bwd_flops(cfg)
    cols_ms = trace["bwd_cols"][1] / max(trace["bwd_cols"][0], 1)
    ach = cols_flops / (cols_ms * 1e-3) / 1e12
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    mtok = tok / (ms * 1e-3) / 1e6
    if tensor:
        # fp16 operands: the dense fp16 tensor peak equals the bf16 one (cuBLAS bf16, measured)
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS.get("bf16_tflops", 1590.0)))
        roof_bound, roof_src = "tensor", "%s (MEASURED_PEAKS.json bf16_tflops; fp16 has the same rate)" % peak_kind
    else:
        peak = FP32_ALU_TFLOPS
        roof_bound, roof_src = "alu", "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz"
    out = {"stage": "backward", "metric": "SSD chunked-scan backward Mtokens/s", "value": mtok,
           "unit": "Mtokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
           "higher_is_better": True, "dtype": "%s-in/f32" % cfg.dtype, "data": "synthetic (seeded)",
           "config": {"workload": cfg.name, "batch": b, "seqlen": L, "heads": H, "head_dim": P, "state_dim": N,
                      "groups": G, "chunk_size": Q, "in_dtype": cfg.dtype, "grads": "f32",
                      "init_state": cfg.init == "normal", "l2": "rotating %d input/gradient sets" % nsets},
           "roofline": {"bound": roof_bound, "kernel": "bwd_cols", "achieved": ach, "peak": peak,
                        "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                        "kernel_ms_avg": cols_ms, "kernel_flops": cols_flops, "peak_source": roof_src,
                        "shares": {k: round(v[1] / max(tot_ms, 1e-12), 4) for k, v in trace.items()},
                        "path": {"algorithmic_flops": flops, "algorithmic_bytes": nbytes,
                                 "compute_ms": flops / (peak * 1e12) * 1e3,
                                 "hbm_ms": nbytes / (hbm * 1e9) * 1e3,
                                 "frac": flops / (peak * 1e12) * 1e3 / ms}},
           "bwd_path": path, "simt": simt,
           "clocks": clk, "gpu_launches": int(sum(v[0] for v in trace.values()))}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_bwd(cfg)
    return out


def cpu_baseline_bwd(cfg, budget_s=5.0):
    """The oracle's backward on a bounded sample: every head of batch 0 over
    the full sequence (one thread per head), token-heads scaled to tokens."""
    import oracle
    from state_space_sequence_scan_b200.inputs import make_grad_inputs
    inp = make_scan_inputs(cfg)
    gr = make_grad_inputs(cfg)
    hs = cfg.nheads
    hpg = cfg.nheads // cfg.ngroups
    sub = {k: v for k, v in inp.items()}
    sub["x"] = inp["x"][:1, :, :hs]
    sub["dt_raw"] = inp["dt_raw"][:1, :, :hs]
    for k in ("dt_bias", "A", "D"):
        sub[k] = inp[k][:hs]
    gsel = [h // hpg for h in range(hs)]
    sub["B"] = inp["B"][:1][:, :, gsel]
    sub["C"] = inp["C"][:1][:, :, gsel]
    sub["init_state"] = None if inp["init_state"] is None else inp["init_state"][:1, :hs]
    reps, t0 = 0, time.perf_counter()
    while True:                        # repeated until about 5 s of CPU time have passed
        oracle.scan_bwd(sub["x"], sub["dt_raw"], sub["dt_bias"], sub["A"], sub["B"], sub["C"], sub["D"],
                        gr["dy"][:1, :, :hs], dfinal=gr["dfinal"][:1, :hs], init_state=sub["init_state"])
        reps += 1
        sec = time.perf_counter() - t0
        if sec >= budget_s or reps >= 1000:
            break
    return {"value": reps * cfg.seqlen * hs / cfg.nheads / sec / 1e6, "unit": "Mtokens/s",
            "cores": min(hs, os.cpu_count()), "kind": "oracle",
            "sample": "%d heads of batch 0 (each its own group), full seqlen %d, x%d repeats (%.1f s); "
                      "tokens counted as token-heads / heads" % (hs, cfg.seqlen, reps, sec)}


def kernel_bytes(cfg, name, states=False) -> float:
    b, L, H, P, N, G = cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, cfg.state_dim, cfg.ngroups
    e = 4 if cfg.dtype == "f32" else 2
    tok = b * L
    x, bc, dt, y = tok * H * P * e, tok * G * N * e, tok * H * 4, tok * H * P * 4
    st = b * H * N * P * 4
    if name.endswith("chunk_out"):
        return float(x + 2 * bc + y) + (states_bytes(cfg) if states and name.startswith("tc_") else 0.0)
    if name.endswith("chunk_state") or name.endswith("unit_state"):
        return float(x + bc + dt)
    if name.endswith("state_pass"):
        return float(st * (2 if cfg.init == "normal" else 1))
    return scan_bytes(cfg, states)


def cpu_baseline_scan(cfg, budget_s=12.0):
    """The oracle as it stands, on this host's cores, on a bounded sample:
    whole sequences of a subset of (batch, head) chains, repeated until the
    budget is used.  Returned in the metric's unit (tokens of all heads)."""
    import numpy as np
    import oracle
    inp = make_scan_inputs(cfg)
    cores = os.cpu_count() or 1
    H = cfg.nheads
    G = cfg.ngroups
    # a sample of heads of batch 0 (each chain is independent)
    nh = min(H, max(1, cores))
    heads = list(range(nh))
    sub = dict(x=inp["x"][:1, :, :nh], dt_raw=inp["dt_raw"][:1, :, :nh], dt_bias=inp["dt_bias"][:nh],
               A=inp["A"][:nh], D=inp["D"][:nh])
    gsel = [h // (H // G) for h in heads]
    sub["B"] = inp["B"][:1, :, gsel]
    sub["C"] = inp["C"][:1, :, gsel]
    sub["init_state"] = None if inp["init_state"] is None else inp["init_state"][:1, :nh]
    # G' = nh: every sampled head reads its own group's B, C
    t0 = time.time()
    reps = 0
    while True:
        oracle.scan(sub["x"], sub["dt_raw"], sub["dt_bias"], sub["A"], sub["B"], sub["C"], sub["D"],
                    init_state=sub["init_state"], nthreads=cores)
        reps += 1
        if time.time() - t0 >= budget_s or reps >= 200:
            break
    el = time.time() - t0
    token_heads = reps * cfg.seqlen * nh
    mtok = token_heads / H / el / 1e6
    return dict(value=mtok, unit="Mtokens/s", cores=cores, kind="oracle",
                sample="%d of %d heads of batch 0, full seqlen %d, x%d repeats (%.1f s); tokens counted as "
                       "token-heads / heads" % (nh, H, cfg.seqlen, reps, el), seconds=el)


def cpu_baseline_step(cfg, budget_s=12.0):
    import numpy as np
    import oracle
    cores = os.cpu_count() or 1
    rows = max(1, min(cfg.batch, 16))
    c2 = cfg.with_(batch=rows)
    inp = make_step_inputs(c2, steps=8)
    st = inp["state"].double().numpy().copy()
    t0 = time.time()
    n = 0
    while True:
        t = n % 8
        oracle.step(inp["x"][t], inp["dt_raw"][t], inp["dt_bias"], inp["A"], inp["B"][t], inp["C"][t], inp["D"],
                    st, nthreads=cores)
        n += 1
        if time.time() - t0 >= budget_s or n >= 2000:
            break
    el = time.time() - t0
    gbs = step_bytes(c2) * n / el / 1e9
    return dict(value=gbs, unit="GB/s", cores=cores, kind="oracle",
                sample="%d of %d batch rows, %d steps (%.1f s); algorithmic state bytes per step" %
                       (rows, cfg.batch, n, el), seconds=el)


def run_reference(args, ws, rank):
    """--impl reference: the fp64 CPU oracle (this method has no other
    reference implementation) timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    cfg, is_step = pick(args.workload)
    steps, warm = args.steps, args.warmup
    budget = max(2.0, min(60.0, 6.0 * steps / max(steps + warm, 1)))
    if is_step:
        cb = cpu_baseline_step(cfg, budget_s=budget)
        value, unit, hib = cb["value"], "GB/s", True
        ms = step_bytes(cfg) / (cb["value"] * 1e9) * 1e3
        dtype = "f64"
    else:
        cb = cpu_baseline_scan(cfg, budget_s=budget)
        value, unit, hib = cb["value"], "Mtokens/s", True
        ms = cfg.tokens / (cb["value"] * 1e6) * 1e3
        dtype = "f64"
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": steps, "warmup": warm,
            "ms_per_step": ms, "higher_is_better": hib, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
            "data": "synthetic", "impl": "reference", "config": workload_config(cfg, is_step),
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def pick(name):
    if name in SCAN_CONFIGS:
        return SCAN_CONFIGS[name], False
    if name in STEP_CONFIGS:
        return STEP_CONFIGS[name], True
    raise SystemExit("unknown workload %s (scan: %s; decode: %s)" % (name, list(SCAN_CONFIGS), list(STEP_CONFIGS)))


def workload_config(cfg, is_step, nsets=None, states=False, packed=False):
    if is_step:
        c = {"workload": cfg.name, "batch": cfg.batch, "heads": cfg.nheads, "head_dim": cfg.head_dim,
             "state_dim": cfg.state_dim, "groups": cfg.ngroups, "state_dtype": "f32", "in_dtype": cfg.dtype,
             "l2": "state %.0f MB > L2, streamed every step" % (cfg.batch * cfg.nheads * cfg.state_dim *
                                                              cfg.head_dim * 4 / 1e6)}
    else:
        c = {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen, "heads": cfg.nheads,
             "head_dim": cfg.head_dim, "state_dim": cfg.state_dim, "groups": cfg.ngroups,
             "chunk_size": cfg.chunk_size, "in_dtype": cfg.dtype, "y_dtype": "f32",
             "init_state": cfg.init != "zero"}
        if nsets is not None:
            one = scan_bytes(cfg, states)
            c["l2"] = ("rotating %d input/output sets (%.0f MB > 2x L2)" % (nsets, nsets * one / 1e6)
                       if nsets > 1 else "inputs %.0f MB > L2" % (one / 1e6))
        if states:
            c["chunk_states"] = "[b, %d, H, N, P] f32 written every step" % math.ceil(cfg.seqlen / cfg.chunk_size)
        if packed:
            c["packed"] = "documents of about 512 tokens per row (seq_idx); e2e leg unpacked"
    return c


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c3_long",
                    help="the headline workload (default: the largest single-GPU scan, c3_long)")
    ap.add_argument("--also", default="c1_130m,c2_2p7b",
                    help="comma-separated scan workloads timed in the same run and nested in the line "
                         "under 'configs' ('none' for none)")
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--no-decode", action="store_true", help="skip the decode figure on the scan line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="leave the backward (ssd_chunk_scan_bwd) line out of the default scan run")
    ap.add_argument("--backward-workload", default="c1_130m",
                    help="the workload of the nested backward line")
    ap.add_argument("--chunk-states", action="store_true",
                    help="the scan also writes the chunk-boundary states [b, nc, H, N, P] (f32) every step")
    ap.add_argument("--packed", action="store_true",
                    help="rows packed with documents of about 512 tokens (seq_idx)")
    ap.add_argument("--stage", default="scan", choices=["scan", "conv1d", "gated_norm", "backward", "conv_scan"],
                    help="time one of the steps either side of the scan, the backward, or the conv and the "
                         "scan in both arrangements instead (one GPU)")
    ap.add_argument("--no-conv-scan", action="store_true",
                    help="leave the conv + scan arrangements (split, combined) out of the default scan run")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    ws, rank, local = init_dist()
    try:
        if args.impl == "reference":
            run_reference(args, ws, rank)
            return
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (the product path has no CPU fallback)")
        from state_space_sequence_scan_b200 import ssd
        ssd.load_library()
        peaks, peak_kind = load_peaks()
        cfg, is_step = pick(args.workload)
        if args.stage != "scan" and not is_step:
            if rank == 0:
                fn = {"backward": bench_backward, "conv_scan": bench_conv_scan}.get(args.stage, bench_stage)
                print(json.dumps(fn(cfg, args, local, peaks, peak_kind)), flush=True)
            return
        if is_step:
            r = bench_step(cfg, args, ws, rank, local)
        else:
            r = bench_scan(cfg, args, ws, rank, local)
        out = finish(cfg, is_step, r, args, ws, rank, peaks, peak_kind)
        del r
        torch.cuda.empty_cache()
        if not is_step:
            # the other scan workloads, each a full record nested under "configs"
            extra = [w for w in args.also.split(",") if w and w != "none" and w != cfg.name]
            nested = {}
            for wname in extra:
                wcfg, wstep = pick(wname)
                if wstep:
                    continue
                wr = bench_scan(wcfg, args, ws, rank, local)
                line = finish(wcfg, False, wr, args, ws, rank, peaks, peak_kind, sub=True)
                del wr
                torch.cuda.empty_cache()
                if line is not None:
                    if ws == 1 and not args.no_cpu_baseline:
                        cb = cpu_baseline_scan(wcfg, budget_s=5.0)
                        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
                    nested[wname] = line
            if out is not None and nested:
                out["configs"] = nested
        if not is_step and not args.no_decode:
            dcfg = STEP_CONFIGS["c4_decode"]
            dr = bench_step(dcfg, args, ws, rank, local)
            dline = finish(dcfg, True, dr, args, ws, rank, peaks, peak_kind, sub=True)
            if out is not None:
                out["decode"] = dline
        if not is_step and ws == 1 and not args.no_backward and out is not None:
            bcfg, _ = pick(args.backward_workload)
            out["backward"] = bench_backward(bcfg, args, local, peaks, peak_kind)
        if not is_step and ws == 1 and not args.no_conv_scan and out is not None and cfg.dtype == "bf16":
            out["conv_scan"] = bench_conv_scan(cfg, args, local, peaks, peak_kind)
        if rank == 0 and out is not None:
            if ws == 1 and not args.no_cpu_baseline:
                cb = cpu_baseline_step(cfg) if is_step else cpu_baseline_scan(cfg)
                out["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
            print(json.dumps(out), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def finish(cfg, is_step, r, args, ws, rank, peaks, peak_kind, sub=False):
    ms_step = r["ms"] / args.steps
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    name, n, kms = dominant(r["trace"])
    avg = kms / max(n, 1)
    if is_step:
        value = ws * r["bytes"] / (ms_step * 1e-3) / 1e9
        unit = "GB/s"
        kb = r["bytes"]
        dtype = "f32"
        e2e_val = ws * r["bytes"] / (r["e2e"]["ms_per_step"] * 1e-3) / 1e9
    else:
        value = ws * r["tokens"] / (ms_step * 1e-3) / 1e6
        unit = "Mtokens/s"
        kb = kernel_bytes(cfg, name, args.chunk_states) if name else r["bytes"]
        dtype = "f32" if cfg.dtype == "f32" else "bf16-in/f32"
        e2e_val = ws * r["tokens"] / (r["e2e"]["ms_per_step"] * 1e-3) / 1e6
    achieved = kb / (avg * 1e-3) / 1e9 if avg > 0 else None
    traffic, traffic_src = measured_traffic(cfg.name, name) if name else (None, None)
    roof = {"bound": "hbm", "kernel": name, "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": (achieved / hbm) if achieved else None, "traffic": traffic, "traffic_source": traffic_src,
            "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "kernel_ms_avg": avg, "kernel_bytes": kb,
            "shares": {k: round(v[1] / max(sum(x[1] for x in r["trace"].values()), 1e-12), 4)
                       for k, v in r["trace"].items()}}
    if not is_step:
        t_mem = r["bytes"] / (hbm * 1e9)
        t_flop = r["flops"] / (float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * 1e12)
        t_roof = max(t_mem, t_flop)
        roof["path"] = {"roofline_ms": t_roof * 1e3, "ms_per_step": ms_step,
                        "frac": t_roof * 1e3 / ms_step, "bound": "hbm" if t_mem >= t_flop else "tensor",
                        "algorithmic_bytes": r["bytes"], "algorithmic_flops": r["flops"]}
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype, "data": "synthetic (seeded; shapes/distributions of the workload)",
            "config": workload_config(cfg, is_step, r.get("nsets"), (not is_step) and args.chunk_states,
                                      (not is_step) and args.packed),
            "roofline": roof, "clocks": r["clocks"],
            "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": r["e2e"]["h2d"],
                    "d2h_bytes_per_step": r["e2e"]["d2h"], "ms_per_step": r["e2e"]["ms_per_step"],
                    **({"pipelined": r["e2e"]["pipelined"]} if "pipelined" in r["e2e"] else {})},
            "gpu_launches": r["launches"]}
    if sub:
        for k in ("metric", "n_gpus", "steps", "warmup", "higher_is_better", "scaling", "vs_baseline", "data"):
            line.pop(k, None)
    return line if rank == 0 else None


if __name__ == "__main__":
    main()
