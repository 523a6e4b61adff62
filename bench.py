#!/usr/bin/env python
"""Benchmark of the SSD layer scan on B200: one JSON line on rank 0.

Workload (one "step"): the chunked scan forward of a 2.7B-scale Mamba-2 layer -- batch 4,
4096 tokens, 80 heads of headdim 64, state 128, 1 group, chunk 256, bf16 x/B/C with fp32
accumulation, final states returned -- i.e. all four kernels of the chunked path (dA cumsum,
chunk state, state passing, chunk scan).  The recurrent decode update (batch 128, 80 heads,
64 x 128 fp32 state, one token per call) is timed in the same run and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Timing: W untimed warm-up steps, then K steps each bracketed by CUDA events on the launching
stream, with a 256 MB buffer written between steps (outside the events) to flush L2; inputs
already resident in HBM.  Per-kernel times come from events the library records between its
kernels (ssd_chunk_scan_fwd_staged).  Under torchrun each rank runs its own replica (weak
scaling, no data-path collective) and the time is the max over ranks.  --impl reference times
the float64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mamba_ssd_layer_scan_b200 import configs, inputs  # noqa: E402

KERNELS = ("chunk_cumsum", "chunk_state", "state_passing", "chunk_scan")
# Kernels of one ssd_chunk_scan_bwd call with dfinal and dinit, no initial state: a zero fill;
# the reversed tensor-core scan (3 gathers, dt shift, 4 scan kernels) and dinit; the dB scan and
# the dC scan (cumsum, tensor-core chunk state, state passing, chunk scan, group sum each); the
# final-state dot product, the token and decay kernels and the batch sum of dA and dD.
BWD_KERNELS = 1 + 8 + 1 + 5 + 5 + 4
KERNEL_SOURCES = {
    "chunk_cumsum": ["chunk_cumsum.cu"],
    "chunk_state": ["chunk_tc.cu", "sm100.cuh"],
    "state_passing": ["state_passing.cu"],
    "chunk_scan": ["chunk_tc.cu", "sm100.cuh"],
    "state_update": ["state_update.cu"],
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ work model
def work_model(w):
    """Algorithmic bytes and flops per launch of each kernel, and for the whole step.

    Algorithmic bytes are the compulsory traffic of the method: x, B, C and dt read, y written,
    the initial state read and the final state written, each counted once (element size e for
    x/B/C/y, 4 for float32).  Each kernel's share is the part of that traffic it must move:
    the cumsum kernel reads dt; the chunk-state kernel reads x, B and dt; the state-passing
    kernel reads the initial state and writes the final state; the chunk-scan kernel reads x, B,
    C and dt and writes y.  What a
    kernel moves beyond that is workspace traffic, reported separately as "ws_bytes": the
    per-chunk float32 states (written by the chunk-state kernel, read by state passing), the
    bf16 states entering each chunk (written by state passing, read by the chunk scan), and the
    chunk-local cumsum rows (written by the cumsum kernel, read by the two tensor-core kernels;
    the dt rows it re-lays out per chunk stand in for the dt those kernels count).  Flops count the dense Q x Q intra-chunk product as the method materialises it,
    plus the chunk-state and off-chunk products (2NP each per token-head) and C B^T once per
    group (2QN per token-group); "flops_causal" counts only the causal half of the Q x Q block."""
    b, L, H, P, N, G, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk
    c = -(-L // Q)
    e = 2 if w.dtype == "bf16" else 4
    x = b * L * H * P * e
    y = x
    bc = b * L * G * N * e
    dt = b * L * H * 4
    cs = b * c * H * Q * 4            # cs rows; the dt rows re-laid out per chunk are the same size
    st = b * c * H * P * N            # elements of the per-chunk states
    fin = b * H * P * N * 4
    init = fin if w.init_state else 0
    k = {
        "chunk_cumsum": {"bytes": dt, "ws_bytes": 2 * cs, "flops": 0},
        "chunk_state": {"bytes": x + bc + dt, "ws_bytes": cs + st * 4,
                        "flops": 2 * b * L * H * P * N},
        "state_passing": {"bytes": fin + init, "ws_bytes": cs // Q + st * 4 + st * 2,
                          "flops": 0},
        "chunk_scan": {"bytes": x + 2 * bc + dt + y, "ws_bytes": cs + st * 2,
                       "flops": b * L * H * (2 * Q * P + 2 * N * P) + b * L * G * 2 * Q * N,
                       "flops_causal": b * L * H * ((Q + 1) * P + 2 * N * P)
                       + b * L * G * (Q + 1) * N},
    }
    total = {"bytes": x + 2 * bc + dt + y + fin + init,
             "flops": b * L * H * (2 * Q * P + 4 * N * P) + b * L * G * 2 * Q * N,
             "flops_causal": b * L * H * ((Q + 1) * P + 4 * N * P) + b * L * G * (Q + 1) * N}
    return k, total


def decode_bytes(w):
    e = 2 if w.dtype == "bf16" else 4
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    return 2 * b * H * P * N * 4 + 2 * b * H * P * e + 2 * b * G * N * e + b * H * 4


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "mamba_ssd_layer_scan_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """dram bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == workload and f[1] == kernel:
            return int(f[2]) if f[3] == source_hash(kernel) else None
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples of one GPU while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, nvml_index):
        self.idx = nvml_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def nvml_index(torch, dev):
    try:
        return torch.cuda._get_nvml_device_index(dev)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[dev])
            except ValueError:
                pass
        return dev


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks of the default process group (the value itself when
    there is no group).  Timing of a multi-GPU step is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def scaled_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: every rank processed `units_per_rank` in (max-over-ranks) `seconds`."""
    return world * units_per_rank / seconds


# ------------------------------------------------------------------ CPU oracle timing
def time_oracle(w, inp, target_s, max_pairs=None):
    """Run the float64 oracle on (batch, head) slices of the full sequence until about
    target_s seconds have passed; returns (tokens/s scaled to whole-layer tokens, sample text,
    threads)."""
    import oracle
    threads = oracle.num_threads()
    pairs_all = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    rng = np.random.default_rng(0)
    order = rng.permutation(len(pairs_all))
    done, t0 = 0, time.perf_counter()
    while done == 0 or (time.perf_counter() - t0 < target_s and done < len(pairs_all)):
        batch = [pairs_all[i] for i in order[done:done + threads]]
        if max_pairs is not None:
            batch = batch[:max(0, max_pairs - done)]
            if not batch:
                break
        oracle.ssd_scan_pairs(inp, batch)
        done += len(batch)
    el = time.perf_counter() - t0
    tokens = done * w.seqlen / w.nheads
    sample = (f"{done} of {w.batch * w.nheads} (batch, head) slices over the full "
              f"{w.seqlen}-token sequence, float64 recurrence; tokens/s = slices * L / H / s")
    return tokens / el, sample, threads, el


# ------------------------------------------------------------------ reference arm
def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = inputs.make_inputs(w)
    import oracle
    threads = oracle.num_threads()
    # one step = one bounded sample: `threads` slices (about 1-3 s of host work)
    steps = []
    for i in range(args.warmup + args.steps):
        v, sample, thr, el = time_oracle(w, inp, target_s=0.0, max_pairs=threads)
        if i >= args.warmup:
            steps.append((v, el))
    value = len(steps) / sum(1.0 / v for v, _ in steps)   # tokens over total time
    ms = 1e3 * statistics.mean(el for _, el in steps)
    line = {
        "impl": "reference", "metric": "ssd_chunk_scan_fwd_tokens_per_s", "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups,
                   "chunk": w.chunk, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                         "sample": f"per step: {thr} (batch, head) slices over the full "
                                   f"{w.seqlen}-token sequence, float64 recurrence; "
                                   "tokens/s = slices * L / H / s"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ forward timing
def device_inputs(torch, w, inp, dev):
    xdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in
            dict(x=inp.x, dt=inp.dt, A=inp.A, B=inp.B, C=inp.C, D=inp.D).items()}
    host["x"], host["B"], host["C"] = (host[k].to(xdt) for k in ("x", "B", "C"))
    if inp.init is not None:
        host["init"] = torch.from_numpy(np.ascontiguousarray(inp.init))
    return host, {k: v.to(dev) for k, v in host.items()}


def time_forward(ssd, torch, w, t, dev, stream, K, warmup, flush, barrier=lambda: None,
                 before_timing=None):
    """K plain ssd_chunk_scan_fwd calls, each bracketed by CUDA events on the launching stream
    with the L2 flush written before it (outside the events), after `warmup` untimed calls;
    then K staged calls (events between the kernels) for the per-kernel times.  Returns
    (per-step ms, staged per-step ms, per-kernel ms lists, wall seconds of the timed loop)."""
    shape = ssd.make_shape(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                           ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32)
    ws = ssd.new_workspace(shape, w.chunk, dev)
    y = torch.empty_like(t["x"])
    final = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                        device=dev)
    init = t.get("init")

    def fwd(events=None):
        ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], w.chunk,
                           init_state=init, y=y, final_state=final, workspace=ws,
                           stage_events=events)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for row in ev:            # create the underlying CUDA events before handing them over
        for e in row:
            e.record(stream)
    for _ in range(warmup):
        flush.fill_(1.0)
        fwd()
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK, "in-kernel timeout during warm-up"
    if before_timing:
        before_timing(fwd)
    # The timed steps are plain calls: events recorded between the four kernels would keep each
    # kernel from starting while its predecessor drains (programmatic dependent launch), so the
    # per-kernel breakdown comes from a second, staged pass below.
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(K):
        flush.fill_(1.0)
        ev_step[i][0].record(stream)
        fwd()
        ev_step[i][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    wall = time.perf_counter() - wall0
    assert ssd.workspace_status(ws) == ssd.SSD_OK, "in-kernel timeout during timing"
    for i in range(K):
        flush.fill_(1.0)
        fwd(ev[i])
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK, "in-kernel timeout during the staged pass"
    step_ms = [a.elapsed_time(e) for a, e in ev_step]
    staged_ms = [ev[i][0].elapsed_time(ev[i][4]) for i in range(K)]
    kern_ms = {name: [ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)]
               for j, name in enumerate(KERNELS)}
    return step_ms, staged_ms, kern_ms, wall, (ws, y, final)


def time_graph(ssd, torch, w, t, stream, K, flush):
    """The same step captured once into a CUDA graph (ssd.CapturedScan) and replayed: K
    replays, each bracketed by CUDA events with the L2 flush written before it (outside the
    events).  Returns the mean ms per replay."""
    cap = ssd.CapturedScan(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], w.chunk,
                           init_state=t.get("init"))
    for _ in range(3):
        flush.fill_(1.0)
        cap.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for a, b in ev:
        flush.fill_(1.0)
        a.record(stream)
        cap.replay()
        b.record(stream)
    torch.cuda.synchronize()
    assert ssd.workspace_status(cap.workspace) == ssd.SSD_OK, "graph replay status"
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def kernel_rooflines(w, staged_ms, kern_ms, hbm, tc_peak):
    """Per kernel: mean time, share of the staged step, achieved GB/s on its algorithmic bytes
    and on all the bytes it moves (algorithmic + workspace), TFLOP/s, the fractions of the
    measured peaks, and which roof bounds it at its algorithmic intensity."""
    kmodel, _ = work_model(w)
    out = {}
    for name in KERNELS:
        ms = statistics.mean(kern_ms[name])
        m = kmodel[name]
        sec = ms / 1e3
        gbs = m["bytes"] / sec / 1e9
        gbs_moved = (m["bytes"] + m["ws_bytes"]) / sec / 1e9
        tfs = m["flops"] / sec / 1e12
        t_hbm = m["bytes"] / (hbm * 1e9)
        t_tc = m["flops"] / (tc_peak * 1e12)
        out[name] = {"ms": ms, "share": ms / statistics.mean(staged_ms), "gbs": gbs,
                     "frac_hbm": gbs / hbm, "gbs_moved": gbs_moved,
                     "frac_hbm_moved": gbs_moved / hbm, "tflops": tfs,
                     "frac_tensor": tfs / tc_peak,
                     "bound": "tensor" if t_tc > t_hbm else "hbm",
                     "alg_bytes": m["bytes"], "ws_bytes": m["ws_bytes"], "alg_flops": m["flops"]}
    return out


def tensor_core_summary(w, kernels, tc_peak, hbm):
    kmodel, _ = work_model(w)
    tc_ms = kernels["chunk_state"]["ms"] + kernels["chunk_scan"]["ms"]
    tc_flops = kmodel["chunk_state"]["flops"] + kmodel["chunk_scan"]["flops"]
    tc_bytes = kmodel["chunk_state"]["bytes"] + kmodel["chunk_scan"]["bytes"]
    tf = tc_flops / (tc_ms / 1e3) / 1e12
    gb = tc_bytes / (tc_ms / 1e3) / 1e9
    return {"tflops": tf, "frac_of_bf16_peak": tf / tc_peak, "gbs": gb, "frac_hbm": gb / hbm,
            "ms": tc_ms, "flops": tc_flops, "alg_bytes": tc_bytes,
            "kernels": ["chunk_state", "chunk_scan"]}


def step_summary(w, ms_per_step, hbm, tc_peak):
    _, total = work_model(w)
    sec = ms_per_step / 1e3
    return {"alg_bytes": total["bytes"], "alg_flops": total["flops"],
            "alg_flops_causal": total["flops_causal"],
            "gbs_compulsory": total["bytes"] / sec / 1e9,
            "frac_hbm": total["bytes"] / sec / 1e9 / hbm,
            "tflops_dense": total["flops"] / sec / 1e12,
            "tflops_causal": total["flops_causal"] / sec / 1e12,
            "frac_tensor_dense": total["flops"] / sec / 1e12 / tc_peak}


# ------------------------------------------------------------------ our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-steps", type=int, default=None)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = configs.SSD_2P7B
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    from mamba_ssd_layer_scan_b200 import ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    # ---- inputs for the scan (same seeded draw on every rank: weak-scaling replicas)
    inp = inputs.make_inputs(w)
    xdt = torch.bfloat16
    host, t = device_inputs(torch, w, inp, dev)
    pinned = {k: v.pin_memory() for k, v in host.items()}
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    K = args.steps

    sampler = ClockSampler(nvml_index(torch, local)) if rank == 0 else None

    def start_clocks(fwd):
        if sampler:
            sampler.start()
            t_pre = time.perf_counter()
            while time.perf_counter() - t_pre < 0.6:      # load the GPU while sampling starts
                fwd()
            torch.cuda.synchronize()

    step_ms, staged_ms, kern_ms, wall, (ws, y, final) = time_forward(
        ssd, torch, w, t, dev, stream, K, args.warmup, flush, barrier, start_clocks)
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / K
    tokens_per_step = w.batch * w.seqlen
    value = scaled_throughput(tokens_per_step * K, world, total_ms / 1e3)

    # ---- the other forward workloads of the layer scan: the ~370M layer (batch 2 x 2048 x 24
    # heads) and the long-context case (1 x 65536 tokens, 32 heads, 8 groups, initial state)
    extra = {}
    for wx in (configs.SSD_370M, configs.SSD_LONG):
        _, tx = device_inputs(torch, wx, inputs.make_inputs(wx), dev)
        Kx = max(10, min(K, 100))
        sx, stx, kx, _, _ = time_forward(ssd, torch, wx, tx, dev, stream, Kx, args.warmup, flush)
        gx = time_graph(ssd, torch, wx, tx, stream, Kx, flush)
        extra[wx.name] = (wx, Kx, sx, stx, kx, gx)
        del tx
    graph_ms = time_graph(ssd, torch, w, t, stream, max(10, min(K, 100)), flush)

    # ---- end to end through the C ABI with host buffers: every step copies its inputs from
    # pinned host memory, runs the scan through the public API and copies y and the final state
    # back.  Upload, compute and download run on three streams with two device buffer sets, so
    # step i+1's upload and step i-1's download overlap step i's compute (the two copy
    # directions use separate copy engines); every copy of every step is inside the timed region.
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    f_host = [torch.empty(final.shape, dtype=final.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_host[0].numel() * y_host[0].element_size() + f_host[0].numel() * f_host[0].element_size()
    K_e2e = max(3, min(K, 20))
    s_up = torch.cuda.Stream(dev)
    s_dn = torch.cuda.Stream(dev)
    ins = [t, {k: torch.empty_like(v) for k, v in t.items()}]
    outs = [(y, final), (torch.empty_like(y), torch.empty_like(final))]
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_dn = [torch.cuda.Event() for _ in range(2)]
    for ev in ev_up + ev_cmp + ev_dn:
        ev.record(stream)

    def e2e_step(i):
        j = i % 2
        s_up.wait_event(ev_cmp[j])            # step i-2's compute is done with input set j
        with torch.cuda.stream(s_up):
            for k, v in pinned.items():
                ins[j][k].copy_(v, non_blocking=True)
        ev_up[j].record(s_up)
        stream.wait_event(ev_up[j])
        stream.wait_event(ev_dn[j])            # step i-2's download is done with output set j
        ssd.chunk_scan_fwd(ins[j]["x"], ins[j]["dt"], ins[j]["A"], ins[j]["B"], ins[j]["C"],
                           ins[j]["D"], w.chunk, y=outs[j][0], final_state=outs[j][1],
                           workspace=ws, stream=stream)
        ev_cmp[j].record(stream)
        s_dn.wait_event(ev_cmp[j])
        with torch.cuda.stream(s_dn):
            y_host[j].copy_(outs[j][0], non_blocking=True)
            f_host[j].copy_(outs[j][1], non_blocking=True)
        ev_dn[j].record(s_dn)

    for i in range(2):                          # untimed warm-up of the pipeline
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(s_up)
    for i in range(K_e2e):
        e2e_step(i)
    e_end.record(s_dn)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / K_e2e, dev)
    e2e_value = scaled_throughput(tokens_per_step, world, e2e_ms / 1e3)
    assert ssd.workspace_status(ws) == ssd.SSD_OK, "status after the end-to-end steps"

    # ---- decode update at batch 128, 80 heads, 64 x 128 fp32 state
    wd = configs.SSD_DECODE
    gen = torch.Generator(device=dev).manual_seed(wd.seed)
    state = 0.1 * torch.randn((wd.batch, wd.nheads, wd.headdim, wd.dstate), device=dev,
                              generator=gen)
    xd = torch.randn((wd.batch, wd.nheads, wd.headdim), device=dev, generator=gen).to(xdt)
    dtd = torch.nn.functional.softplus(
        torch.randn((wd.batch, wd.nheads), device=dev, generator=gen) - 4).clamp(1e-3, 0.1)
    Bd = (torch.randn((wd.batch, wd.ngroups, wd.dstate), device=dev, generator=gen)
          / wd.dstate ** 0.5).to(xdt)
    Cd = (torch.randn((wd.batch, wd.ngroups, wd.dstate), device=dev, generator=gen)
          / wd.dstate ** 0.5).to(xdt)
    yd = torch.empty_like(xd)
    Kd = args.decode_steps or max(20, K)
    for _ in range(5):
        ssd.state_update(state, xd, dtd, t["A"], Bd, Cd, t["D"], y=yd)
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    d0.record(stream)
    for _ in range(Kd):
        ssd.state_update(state, xd, dtd, t["A"], Bd, Cd, t["D"], y=yd)
    d1.record(stream)
    torch.cuda.synchronize()
    dec_ms = d0.elapsed_time(d1) / Kd

    # ---- the same step with the block's fused steps: dt <- clamp(softplus(dt_raw + bias)) and
    # the output gated by SiLU(z)
    blk = inputs.make_block_inputs(w)
    bz = torch.from_numpy(blk.z).to(dev).to(xdt)
    bdt = torch.from_numpy(blk.dt_raw).to(dev)
    bbias = torch.from_numpy(blk.dt_bias).to(dev)

    def bfwd():
        ssd.chunk_scan_fwd(t["x"], bdt, t["A"], t["B"], t["C"], t["D"], w.chunk, y=y,
                           final_state=final, workspace=bws, z=bz, dt_bias=bbias,
                           dt_softplus=True, dt_limit=blk.dt_limit)

    bshape = ssd.make_shape(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                            ssd.SSD_BF16)
    bopts = ssd.FwdOptions(bz.data_ptr(), bbias.data_ptr(), 1, *blk.dt_limit)
    bws = torch.empty(ssd.lib().ssd_chunk_scan_fwd_ex_workspace_size(
        ctypes.byref(bshape), w.chunk, ctypes.byref(bopts)), dtype=torch.uint8, device=dev)
    for _ in range(3):
        flush.fill_(1.0)
        bfwd()
    torch.cuda.synchronize()
    Kb = max(10, min(K, 50))
    b_ms = []
    for _ in range(Kb):
        flush.fill_(1.0)
        b0 = torch.cuda.Event(enable_timing=True)
        b1 = torch.cuda.Event(enable_timing=True)
        b0.record(stream)
        bfwd()
        b1.record(stream)
        torch.cuda.synchronize()
        b_ms.append(b0.elapsed_time(b1))
    assert ssd.workspace_status(bws) == ssd.SSD_OK, "fused block scan status"
    block_ms = statistics.mean(b_ms)

    # ---- packed variable-length sequences: the 2.7B layer's tokens as 12 uneven sequences
    wv = configs.SSD_VARLEN
    vin = inputs.make_inputs(wv)
    vt = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in
          dict(x=vin.x, dt=vin.dt, A=vin.A, B=vin.B, C=vin.C, D=vin.D, init=vin.init).items()}
    for k in ("x", "B", "C"):
        vt[k] = vt[k].to(xdt)
    vcu = torch.from_numpy(vin.cu_seqlens).to(dev)
    vshape = ssd.make_shape(1, wv.seqlen, wv.nheads, wv.headdim, wv.dstate, wv.ngroups,
                            ssd.SSD_BF16)
    vws = torch.empty(ssd.varlen_workspace_size(vshape, wv.nseq, wv.chunk), dtype=torch.uint8,
                      device=dev)
    vy = torch.empty_like(vt["x"])
    vfin = torch.empty((wv.nseq, wv.nheads, wv.headdim, wv.dstate), dtype=torch.float32,
                       device=dev)

    def vfwd():
        ssd.chunk_scan_varlen_fwd(vt["x"], vt["dt"], vt["A"], vt["B"], vt["C"], vt["D"], vcu,
                                  wv.chunk, init_states=vt["init"], y=vy, final_states=vfin,
                                  workspace=vws)

    for _ in range(3):
        flush.fill_(1.0)
        vfwd()
    torch.cuda.synchronize()
    Kv = max(10, min(K, 50))
    v_ms = []
    for _ in range(Kv):
        flush.fill_(1.0)
        v0 = torch.cuda.Event(enable_timing=True)
        v1 = torch.cuda.Event(enable_timing=True)
        v0.record(stream)
        vfwd()
        v1.record(stream)
        torch.cuda.synchronize()
        v_ms.append(v0.elapsed_time(v1))
    assert ssd.workspace_status(vws) == ssd.SSD_OK, "varlen scan status"
    varlen_ms = statistics.mean(v_ms)

    # ---- backward pass of the same scan (all seven gradients, forward recomputed inside)
    gin = inputs.make_grad_inputs(w)
    gdy = torch.from_numpy(gin.dy).to(dev).to(xdt)
    gdf = torch.from_numpy(gin.dfinal).to(dev)
    gws = torch.empty(ssd.bwd_workspace_size(bshape, w.chunk), dtype=torch.uint8, device=dev)

    def bwd():
        return ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], gdy, w.chunk,
                                  dfinal=gdf, workspace=gws)

    for _ in range(3):
        flush.fill_(1.0)
        bwd()
    torch.cuda.synchronize()
    Kg = max(5, min(K, 20))
    g_ms = []
    for _ in range(Kg):
        flush.fill_(1.0)
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        bwd()
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms.append(g0.elapsed_time(g1))
    assert ssd.workspace_status(gws) == ssd.SSD_OK, "backward status"
    bwd_ms = statistics.mean(g_ms)
    del gws

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---- rooflines
    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops"]
    kernels = kernel_rooflines(w, staged_ms, kern_ms, hbm, tc_peak)
    dom = max(KERNELS, key=lambda n: kernels[n]["ms"])
    kd = kernels[dom]
    if kd["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": kd["tflops"], "peak": tc_peak,
                "unit": "TFLOP/s", "frac": kd["tflops"] / tc_peak}
    else:
        roof = {"bound": "hbm", "achieved": kd["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": kd["gbs"] / hbm}
    roof.update({"kernel": dom, "traffic": profiled_traffic(dom, w.name),
                 "alg_bytes_per_launch": kd["alg_bytes"], "ws_bytes_per_launch": kd["ws_bytes"],
                 "alg_flops_per_launch": kd["alg_flops"],
                 "frac_hbm": kd["frac_hbm"], "frac_tensor": kd["frac_tensor"],
                 "tensor_core_kernels": {n: {"frac_hbm": kernels[n]["frac_hbm"],
                                             "frac_tensor": kernels[n]["frac_tensor"]}
                                         for n in ("chunk_state", "chunk_scan")},
                 "peak_source": (f"{peak_src} (MEASURED_PEAKS.json burst)"
                                 if peak_src == "measured" else "fallback")})
    config_lines = {}
    for name, (wx, Kx, sx, stx, kx, gx) in extra.items():
        msx = max_over_ranks(sum(sx), dev) / Kx
        kern_x = kernel_rooflines(wx, stx, kx, hbm, tc_peak)
        config_lines[name] = {
            "workload": name, "metric": "ssd_chunk_scan_fwd_tokens_per_s",
            "value": scaled_throughput(wx.batch * wx.seqlen, world, msx / 1e3),
            "unit": "tokens/s", "ms_per_step": msx, "steps": Kx,
            "staged_ms_per_step": statistics.mean(stx),
            "step_totals": step_summary(wx, msx, hbm, tc_peak),
            "tensor_core_kernels": tensor_core_summary(wx, kern_x, tc_peak, hbm),
            "kernels": kern_x,
            "graph": {"ms_per_step": gx, "value": wx.batch * wx.seqlen / (gx / 1e3),
                      "how": "the step captured once into a CUDA graph (ssd.CapturedScan), replayed"},
            "l2": "256 MB buffer written between timed steps (outside the events)"}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, sample, thr, el = time_oracle(w, inp, target_s=15.0)
        cpu = {"value": v, "unit": "tokens/s", "cores": thr, "kind": "oracle", "sample": sample,
               "seconds": el}

    dbytes = decode_bytes(wd)
    line = {
        "metric": "ssd_chunk_scan_fwd_tokens_per_s", "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
                   "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups,
                   "chunk": w.chunk, "final_state": True,
                   "l2": "256 MB buffer written between timed steps (outside the events)",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "staged_ms_per_step": statistics.mean(staged_ms),
        "tensor_core_kernels": tensor_core_summary(w, kernels, tc_peak, hbm),
        "step_totals": step_summary(w, ms_per_step, hbm, tc_peak),
        "kernels": kernels,
        "configs": config_lines,
        "graph": {"ms_per_step": graph_ms, "value": tokens_per_step / (graph_ms / 1e3),
                  "unit": "tokens/s",
                  "how": "the step captured once into a CUDA graph (ssd.CapturedScan), replayed; "
                         "L2 flushed between replays (outside the events)"},
        "fused_block": {"workload": w.name + "_gated_softplus_dt",
                        "metric": "ssd_chunk_scan_fwd_ex_tokens_per_s",
                        "value": tokens_per_step / (block_ms / 1e3), "unit": "tokens/s",
                        "ms_per_step": block_ms, "steps": Kb, "kernels_per_step": 5,
                        "extra_bytes_per_step": int(blk.z.size * 2 + blk.dt_raw.size * 8),
                        "l2": "256 MB buffer written before each timed call (outside the events)"},
        "varlen": {"workload": wv.name, "metric": "ssd_chunk_scan_varlen_fwd_tokens_per_s",
                   "value": wv.seqlen / (varlen_ms / 1e3), "unit": "tokens/s",
                   "ms_per_step": varlen_ms, "steps": Kv,
                   "sequence_lengths": np.diff(vin.cu_seqlens).tolist(),
                   "kernels_per_step": 5,
                   "l2": "256 MB buffer written before each timed call (outside the events)"},
        "backward": {"workload": w.name + "_bwd_dfinal",
                     "metric": "ssd_chunk_scan_bwd_tokens_per_s",
                     "value": tokens_per_step / (bwd_ms / 1e3), "unit": "tokens/s",
                     "ms_per_step": bwd_ms, "steps": Kg, "kernels_per_step": BWD_KERNELS,
                     "gradients": ["dx", "ddt", "dA", "dB", "dC", "dD", "dinit"],
                     "l2": "256 MB buffer written before each timed call (outside the events)"},
        "decode": {"workload": wd.name + " (one token's x, B, C and dt repeated every step)",
                   "metric": "ssd_state_update_GBps", "value":
                   dbytes / (dec_ms / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": dec_ms,
                   "frac_hbm": dbytes / (dec_ms / 1e3) / 1e9 / hbm, "bytes_per_step": dbytes,
                   "tokens_per_s": wd.batch / (dec_ms / 1e3), "steps": Kd},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": K_e2e,
                "pipelined": "upload of step i+1 and download of step i-1 overlap step i "
                             "(3 streams, 2 buffer sets)"},
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": 4 * K,
        "wall_s_timed_region": wall,
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": tc_peak, "source": peak_src},
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
