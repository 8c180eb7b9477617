"""Benchmark of the cached causal Conv3D call on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ccv3d|reference]
                    [--workload NAME]

One step is one ccv3d_forward call (the whole hot path: per-call validation,
tensor-map encode, one launch that computes the implicit GEMM with the bias
epilogue and writes new_cache) on the decoder-bottleneck signature
bf16 384->384, 3x3x3, 90x160, 2-frame cache + 1 frame.  Plans are made once
per signature, as a decoder does; the planner's own cost is reported apart.

Metric: effective TFLOP/s = 2*N*Cout*H_o*W_o*Cin*kh*kw*sum_k(o_h-o_l) per
call (active temporal taps only) / time.  Inputs are resident in HBM; the
timed loop rotates over enough independent input/weight/output sets to exceed
the 126 MB L2, so no call finds its operands in L2 from the previous use.
Under torchrun (N > 1) every rank runs an independent replica (weak scaling,
no collective on the data path); time is the max over ranks.

`--impl reference` times the FP64 CPU oracle on the host cores instead, on a
bounded sample of output points of the same call.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from causal_conv3d_video_b200 import synth, workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


def algorithmic(conv, intervals):
    """FLOPs and bytes of one call (active taps only; Z read once, W once,
    out and new_cache written once)."""
    T_o, H_o, W_o = intervals["T_o"], intervals["H_o"], intervals["W_o"]
    tap_frames = sum(intervals["o_h"][k] - intervals["o_l"][k] for k in range(conv.kt))
    flops = 2.0 * conv.N * conv.Cout * H_o * W_o * conv.Cin * conv.kh * conv.kw * tap_frames
    e = 2 if conv.dtype == "bf16" else 4
    z = conv.cache_len + conv.T_x
    keep = min(conv.cache_keep, z)
    nbytes = e * (z * conv.N * conv.H * conv.W * conv.Cin
                  + conv.Cout * conv.Cin * conv.kt * conv.kh * conv.kw
                  + conv.N * T_o * H_o * W_o * conv.Cout
                  + conv.N * keep * conv.H * conv.W * conv.Cin
                  + (conv.Cout if conv.has_bias else 0))
    return flops, nbytes


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_conv3d_video_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(workload_name):
    """DRAM bytes per launch from profiles/traffic.tsv, only if that row was
    captured with the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.tsv")
    if not os.path.exists(path):
        return None
    digest = kernel_source_digest()
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split("\t")
        if len(parts) >= 3 and parts[0] == workload_name and parts[1] == digest:
            return float(parts[2])
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.stamps = []  # host time each sample line arrived

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # NVML start-up can stall the driver for a moment: let the first
            # sample arrive before the timed region begins.
            t0 = time.time()
            while not self.lines and time.time() - t0 < 15 and self.proc.poll() is None:
                time.sleep(0.02)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.stamps.append(time.time())
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self, t0=None, t1=None):
        """Median SM clock, max clock and active throttle reasons of the samples
        (only those that arrived between host times t0 and t1, when given)."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.lines
        if t0 is not None:
            lines = [l for l, t in zip(list(self.lines), list(self.stamps)) if t0 <= t <= t1]
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for name, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------- replicas over ranks
def max_over_ranks(times_ms, device=None):
    """Each rank's timings -> the maximum over all ranks (the job ends when
    its slowest replica ends).  Works on any initialised process group:
    NCCL with a CUDA device, gloo with the CPU."""
    import torch
    import torch.distributed as tdist

    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(flops_per_call, calls_per_rank, max_ms, world):
    """Whole-job TFLOP/s: every rank ran `calls_per_rank` independent calls
    (weak scaling: fixed work per GPU), the job took the slowest rank's time."""
    return world * flops_per_call * calls_per_rank / (max_ms / 1e3) / 1e12


# --------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    from causal_conv3d_video_b200 import ccv3d

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    conv = workloads.WORKLOADS[args.workload]
    t0 = time.perf_counter()
    plan = ccv3d.Plan(ccv3d.desc_for(conv))
    plan_us = (time.perf_counter() - t0) * 1e6
    flops, nbytes = algorithmic(conv, plan.intervals)
    if args.ring:
        nbytes = ring_algorithmic_bytes(conv, plan.intervals, nbytes)
    slots = conv.cache_len + plan.ring_writes()
    dt = torch.bfloat16 if conv.dtype == "bf16" else torch.float32

    # independent operand sets, enough to exceed L2 between two uses of one set
    n_sets = max(2, int(np.ceil(2.0 * L2_BYTES / nbytes)) + 1)
    sets = []
    heads = [0] * n_sets
    for i in range(n_sets):
        inp = synth.conv_inputs(**conv.synth_kwargs(), stream_base=16 * i)
        to = lambda a: None if a is None else torch.from_numpy(a).to(dt).to(dev)
        out, nc = plan.alloc_outputs(dev)
        cache = to(inp["cache"])
        if args.ring:  # the cache frames in a ring of |C| + n_w slots
            ring = torch.zeros((conv.N, slots, conv.H, conv.W, conv.Cin), dtype=dt, device=dev)
            if cache is not None:
                ring[:, :conv.cache_len] = cache
            cache, nc = ring, None
        sets.append((to(inp["x"]), cache, to(inp["w"]), to(inp["bias"]), out, nc))
    stream = torch.cuda.current_stream(dev)

    def step(i):
        x, c, w, b, out, nc = sets[i % n_sets]
        if args.ring:
            heads[i % n_sets] = plan.forward_ring(x, c, slots, heads[i % n_sets], w, b, out, stream)
        else:
            plan.forward(x, c, w, b, out, nc, stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if plan.status() != 0:
        raise RuntimeError("device status after warm-up: %d" % plan.status())

    dist = world > 1
    if dist:
        import torch.distributed as tdist
    calls0 = plan.stats()
    events = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local_rank) as clocks:
        if dist:
            tdist.barrier()
        torch.cuda.synchronize()
        events[0].record(stream)
        for i in range(args.steps):
            step(i)
            events[i + 1].record(stream)
        torch.cuda.synchronize()
        if dist:
            tdist.barrier()
    per = [events[i].elapsed_time(events[i + 1]) for i in range(args.steps)]
    total_ms = events[0].elapsed_time(events[-1])
    calls1 = plan.stats()
    launches = (calls1["tc_path"] + calls1["simt_path"]) - (calls0["tc_path"] + calls0["simt_path"])
    status = plan.status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {status}")

    # ---- end to end through the C ABI with host buffers -------------------
    # Each step uploads its x and cache from pinned host memory, runs the call
    # and reads out and new_cache back to pinned host memory.  Steps are
    # pipelined over three streams with two device buffer sets, as a
    # streaming decoder runs them: step i+1's upload and step i-1's download
    # overlap step i's compute (PCIe is full duplex).
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    if args.ring:
        e2e_steps = 0  # the host-buffer legs run the dense call only
    w0, b0 = sets[0][2], sets[0][3]
    bufs = []
    for i in range(2):
        x, c, _, _, out, nc = sets[i]
        bufs.append((x, c, out, nc))
    x0, c0, out0, nc0 = bufs[0]
    hx = [torch.empty(x0.shape, dtype=dt, pin_memory=True).copy_(x0) for _ in range(2)]
    hc = ([torch.empty(c0.shape, dtype=dt, pin_memory=True).copy_(c0) for _ in range(2)]
          if c0 is not None else [None, None])
    ho = [torch.empty(out0.shape, dtype=dt, pin_memory=True) for _ in range(2)]
    hn = ([torch.empty(nc0.shape, dtype=dt, pin_memory=True) for _ in range(2)]
          if nc0 is not None else [None, None])
    h2d = x0.numel() * x0.element_size() + (c0.numel() * c0.element_size() if c0 is not None else 0)
    d2h = out0.numel() * out0.element_size() + (nc0.numel() * nc0.element_size() if nc0 is not None else 0)
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()

    def e2e_run(steps, start_ev=None, end_ev=None):
        uploaded = [None, None]   # event: buffer i's inputs are on the device
        computed = [None, None]   # event: buffer i's outputs are written
        freed = [None, None]      # event: buffer i's outputs are read back
        if start_ev is not None:
            start_ev.record(stream)
            s_up.wait_stream(stream)
            s_down.wait_stream(stream)
        for i in range(steps):
            k = i % 2
            x, c, out, nc = bufs[k]
            with torch.cuda.stream(s_up):
                if computed[k] is not None:
                    s_up.wait_event(computed[k])  # previous call on this buffer set read x/cache
                x.copy_(hx[k], non_blocking=True)
                if c is not None:
                    c.copy_(hc[k], non_blocking=True)
                uploaded[k] = ev()
                uploaded[k].record(s_up)
            stream.wait_event(uploaded[k])
            if freed[k] is not None:
                stream.wait_event(freed[k])  # out/new_cache of buffer set k were read back
            plan.forward(x, c, w0, b0, out, nc, stream)
            computed[k] = ev()
            computed[k].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(computed[k])
                ho[k].copy_(out, non_blocking=True)
                if nc is not None:
                    hn[k].copy_(nc, non_blocking=True)
                freed[k] = ev()
                freed[k].record(s_down)
        if end_ev is not None:
            stream.wait_stream(s_up)
            stream.wait_stream(s_down)
            end_ev.record(stream)

    e2e_ms = stream_ms = None
    if e2e_steps > 0:
        e2e_run(3)
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            tdist.barrier()
        torch.cuda.synchronize()
        e2e_run(e2e_steps, ea, eb)
        torch.cuda.synchronize()
        e2e_ms = ea.elapsed_time(eb)

        # Streaming decode: the cache stays on the device, each call's new_cache
        # being the next call's cache (two device buffers, ping-pong); only the
        # new frames go up and only the output comes back.  Needs a steady-state
        # signature (new_cache the shape of the cache).
        stream_ms = None
        if c0 is not None and nc0 is not None and tuple(nc0.shape) == tuple(c0.shape):
            caches = [bufs[0][1], bufs[1][1]]

            def stream_run(steps, start_ev=None, end_ev=None):
                uploaded, computed, freed = [None, None], [None, None], [None, None]
                if start_ev is not None:
                    start_ev.record(stream)
                    s_up.wait_stream(stream)
                    s_down.wait_stream(stream)
                for i in range(steps):
                    k = i % 2
                    x, _, out, _ = bufs[k]
                    with torch.cuda.stream(s_up):
                        if computed[k] is not None:
                            s_up.wait_event(computed[k])
                        x.copy_(hx[k], non_blocking=True)
                        uploaded[k] = ev()
                        uploaded[k].record(s_up)
                    stream.wait_event(uploaded[k])
                    if freed[k] is not None:
                        stream.wait_event(freed[k])
                    plan.forward(x, caches[i % 2], w0, b0, out, caches[(i + 1) % 2], stream)
                    computed[k] = ev()
                    computed[k].record(stream)
                    with torch.cuda.stream(s_down):
                        s_down.wait_event(computed[k])
                        ho[k].copy_(out, non_blocking=True)
                        freed[k] = ev()
                        freed[k].record(s_down)
                if end_ev is not None:
                    stream.wait_stream(s_up)
                    stream.wait_stream(s_down)
                    end_ev.record(stream)

            stream_run(3)
            torch.cuda.synchronize()
            if dist:
                tdist.barrier()
            torch.cuda.synchronize()
            stream_run(e2e_steps, ea, eb)
            torch.cuda.synchronize()
            stream_ms = ea.elapsed_time(eb)

    if dist:
        total_ms = max_over_ranks([total_ms], dev)[0]
        if e2e_ms is not None:
            e2e_ms = max_over_ranks([e2e_ms], dev)[0]
        if stream_ms is not None:
            stream_ms = max_over_ranks([stream_ms], dev)[0]

    if rank != 0:
        return None
    peaks = load_peaks()
    avg_launch_s = (sum(per) / len(per)) / 1e3
    achieved = flops / avg_launch_s / 1e12
    peak = peaks["bf16_tflops"]
    value = job_throughput(flops, args.steps, total_ms, world)
    e2e_value = job_throughput(flops, e2e_steps, e2e_ms, world) if e2e_ms else None
    csum = clocks.summary()
    line = {
        "metric": "cached causal Conv3D effective TFLOP/s (bf16), 1 GPU",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": conv.dtype,
        "data": "synthetic (seeded N(0,1) activations, N(0,1/(Cin*27)) weights)",
        "config": {
            "workload": conv.name, "N": conv.N, "Cin": conv.Cin, "Cout": conv.Cout,
            "ksize": [conv.kt, conv.kh, conv.kw], "H": conv.H, "W": conv.W,
            "T_x": conv.T_x, "cache_len": conv.cache_len, "stride": list(conv.stride),
            "pad": list(conv.pad), "dilation": list(conv.dilation),
            "gflop_per_call": round(flops / 1e9, 3), "mb_per_call": round(nbytes / 1e6, 2),
            "l2": f"rotating {n_sets} operand sets of {nbytes / 1e6:.1f} MB "
                  f"({n_sets * nbytes / 1e6:.0f} MB > 126 MB L2)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "plan": "one plan per signature, made before timing",
            "planner_us": round(plan_us, 1),
            "path": "tcgen05" if plan.path["tc"] else "simt",
            "kernel": plan.kernel,
            "tile": [plan.path["tile_m"], plan.path["tile_n"]],
        },
        "us_per_call_median": round(statistics.median(per) * 1e3, 2),
        "roofline": {
            "bound": "tensor" if conv.dtype == "bf16" else "alu",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic_from_profiles(conv.name + ("+ring" if args.ring else "")),
            "peak_source": f"{peaks['source']} (bf16 burst)",
            "hbm_frac_of_measured": round(nbytes / avg_launch_s / 1e9 / peaks["hbm_gbs"], 4),
            "t_star_us": round(max(flops / (peak * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e6, 2),
        },
        "e2e": None if e2e_value is None else {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "steps": e2e_steps,
                "what": "per step: pinned host x+cache -> device, ccv3d_forward, "
                        "out+new_cache -> pinned host; weights resident; steps pipelined "
                        "over upload/compute/download streams"},
        "e2e_stream": None if stream_ms is None else {
            "value": round(job_throughput(flops, e2e_steps, stream_ms, world), 3),
            "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(x0.numel() * x0.element_size()),
            "d2h_bytes_per_step": int(out0.numel() * out0.element_size()),
            "steps": e2e_steps,
            "what": "streaming decode: per step pinned host x -> device, ccv3d_forward with the "
                    "cache threaded on the device (new_cache of step i is the cache of step "
                    "i+1), out -> pinned host; pipelined like e2e"},
        "gpu_launches": int(launches),
        "clocks": csum,
        "memory": {
            "device_workspace_bytes": int(plan.stats()["workspace_bytes"]),
            "status_block_bytes": 256,
            "intermediate_tensors": 0,
            "what": "device memory the library holds besides the caller's x, cache, W, bias, "
                    "out and new_cache: no concatenated [C;X], no per-tap weight slices, no "
                    "accumulation buffer",
        },
    }
    # side measurements: a failure here is reported in the line, never raised
    if world == 1:
        line["quantize_u8"] = _guarded(run_quantize, dev)
        if not args.no_workloads:
            line["workloads"] = run_workloads(dev, peaks)
        if not args.no_sequence:
            line["decode17"] = _guarded(run_sequence, args, dev)
        line["noalloc"] = _guarded(run_noalloc, conv, dev)
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(conv, args.cpu_seconds)
    return line


# ------------------------------------------------------ per-workload legs
# FP32 FFMA peak of the SIMT path, from unit counts and the maximum clock:
# 148 SMs x 128 FP32 lanes x 2 FLOP per FMA x 1.965 GHz.
FP32_FFMA_TFLOPS = round(148 * 128 * 2 * 1.965e9 / 1e12, 2)
FLUSH_BYTES = 256 * 1024 * 1024   # written between calls whose operands fit in L2 many times


def bench_legs():
    """(leg name, Conv, ring) for every config reported beside the headline:
    the fp32 contract call, the bottleneck call and its cache sweep, the two
    720x1280 calls, the edge sweep, the stride-2 cache sweep, the encoder
    stride-2 calls, the decoder's thin RGB output conv, and the ring-buffer
    variants of the bottleneck and stride-2 calls."""
    W = workloads
    legs = [(c.name, c, False) for c in (
        W.C1, W.C2, W.C2_EMPTY, W.C4_C1, W.C3, W.C3B, W.C4_TIME, W.C4_DIL, W.C4_STRIDE,
        W.C4_ODD, W.C6_ST2_TIME, W.C6_ST2, W.C_RGB)]
    for name in sorted(W.WORKLOADS):
        if name.startswith("bf16_192ch_s2_360x640_c") and name != W.C4_STRIDE.name:
            legs.append((name, W.WORKLOADS[name], False))
    legs += [(W.C2.name + "+ring", W.C2, True), (W.C4_STRIDE.name + "+ring", W.C4_STRIDE, True)]
    return legs


def ring_algorithmic_bytes(conv, intervals, nbytes):
    """A ring-buffer call writes only the arriving frames of the new cache."""
    z = conv.cache_len + conv.T_x
    keep = min(conv.cache_keep, z)
    e = 2 if conv.dtype == "bf16" else 4
    return nbytes - e * conv.N * (keep - min(keep, conv.T_x)) * conv.H * conv.W * conv.Cin


def time_leg(conv, ring, dev, peaks, sampler, seconds=0.6, min_calls=20, max_calls=4000):
    """Median device time of one call of `conv` (CUDA events on the launching
    stream, one event pair per call), operands cold in L2: rotated over sets
    whose total exceeds twice the L2, or, for calls under 36 MB, a 256 MB
    buffer written between calls.  Inputs are seeded N(0,1) activations and
    N(0, 1/(Cin*kt*kh*kw)) weights drawn on the device."""
    import torch
    from causal_conv3d_video_b200 import ccv3d

    plan = ccv3d.Plan(ccv3d.desc_for(conv))
    flops, nbytes = algorithmic(conv, plan.intervals)
    if ring:
        nbytes = ring_algorithmic_bytes(conv, plan.intervals, nbytes)
    dt = torch.bfloat16 if conv.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=dev)
    gen.manual_seed(hash(conv.name) & 0xFFFF)
    flush = nbytes < 36e6
    n_sets = 1 if flush else max(2, int(np.ceil(2.0 * L2_BYTES / nbytes)) + 1)
    rnd = lambda shape, sigma: (sigma * torch.randn(shape, generator=gen, device=dev)).to(dt)
    slots = conv.cache_len + plan.ring_writes()
    sets = []
    for _ in range(n_sets):
        x = rnd((conv.N, conv.T_x, conv.H, conv.W, conv.Cin), 1.0)
        w = rnd((conv.Cout, conv.kt, conv.kh, conv.kw, conv.Cin),
                1.0 / np.sqrt(conv.Cin * conv.kt * conv.kh * conv.kw))
        b = rnd((conv.Cout,), conv.sigma_b) if conv.has_bias else None
        out, nc = plan.alloc_outputs(dev)
        if ring:
            cache = rnd((conv.N, slots, conv.H, conv.W, conv.Cin), 1.0)
            nc = None
        else:
            cache = (rnd((conv.N, conv.cache_len, conv.H, conv.W, conv.Cin), 1.0)
                     if conv.cache_len > 0 else None)
        sets.append([x, cache, w, b, out, nc, 0])
    scratch = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    stream = torch.cuda.current_stream(dev)

    def call(i):
        st = sets[i % n_sets]
        x, cache, w, b, out, nc, head = st
        if ring:
            st[6] = plan.forward_ring(x, cache, slots, head, w, b, out, stream)
        else:
            plan.forward(x, cache, w, b, out, nc, stream)

    def run(n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n):
            if flush:
                scratch.fill_(float(i & 7))
            evs[i][0].record(stream)
            call(i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) * 1e3 for a, b in evs]

    run(3)  # warm-up
    if plan.status() != 0:
        raise RuntimeError(f"{conv.name}: device status {plan.status()} after warm-up")
    est_us = statistics.median(run(3))
    n = int(min(max_calls, max(min_calls, seconds / (est_us * 1e-6 + (4e-5 if flush else 0)))))
    t0 = time.time()
    per = run(n)
    t1 = time.time()
    if plan.status() != 0:
        raise RuntimeError(f"{conv.name}: device status {plan.status()} after timing")
    us = statistics.median(per)
    if conv.dtype == "bf16":
        peak, bound_unit = peaks["bf16_tflops"], "bf16 tensor (measured burst)"
    else:
        peak, bound_unit = FP32_FFMA_TFLOPS, "fp32 FFMA (derived: 148 SMs x 128 lanes x 2 x 1.965 GHz)"
    t_flop = flops / (peak * 1e12) * 1e6
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6
    t_star = max(t_flop, t_hbm)
    # the leg runs ~0.6 s of back-to-back calls: a kernel timed inside a long
    # run, for which the sustained (power-capped) tensor peak is the measure
    sustained = peaks.get("bf16_tflops_sustained")
    line = {
        "kernel": plan.kernel, "calls": n, "us_per_call_median": round(us, 2),
        "us_per_call_min": round(min(per), 2),
        "gflop": round(flops / 1e9, 3), "mb": round(nbytes / 1e6, 2),
        "tflops": round(flops / (us * 1e-6) / 1e12, 2),
        "roofline": {
            "bound": ("tensor" if conv.dtype == "bf16" else "alu") if t_flop >= t_hbm else "hbm",
            "t_star_us": round(t_star, 2), "frac": round(t_star / us, 4),
            "peak_flop": peak, "peak_flop_kind": bound_unit, "peak_hbm_gbs": peaks["hbm_gbs"],
            "traffic": traffic_from_profiles(conv.name + ("+ring" if ring else "")),
        },
        "tensor_frac": round(t_flop / us, 4) if conv.dtype == "bf16" else None,
        "frac_of_sustained": (round(max(flops / (sustained * 1e12) * 1e6, t_hbm) / us, 4)
                              if conv.dtype == "bf16" and sustained else None),
        "hbm_frac": round(t_hbm / us, 4),
        "l2": ("256 MB buffer written between calls" if flush
               else f"rotating {n_sets} operand sets ({n_sets * nbytes / 1e6:.0f} MB)"),
        "clocks": sampler.summary(t0, t1),
    }
    if ring:
        line["ring_slots"] = slots
    del sets, scratch
    torch.cuda.empty_cache()
    return line


def run_workloads(dev, peaks):
    """One timed leg per config; a leg that fails reports its error."""
    import torch

    out = {}
    with ClockSampler(dev.index or 0) as sampler:
        for name, conv, ring in bench_legs():
            out[name] = _guarded(time_leg, conv, ring, dev, peaks, sampler)
            torch.cuda.synchronize()
    return out


# ------------------------------------------------- decode-sequence leg
def _guarded(fn, *a):
    """fn(*a), or {"error": ...} if it raised (the headline line still prints)."""
    try:
        return fn(*a)
    except Exception as e:  # noqa: BLE001 -- recorded, not swallowed silently
        import traceback
        traceback.print_exc()
        return {"error": f"{type(e).__name__}: {e}"}


def run_noalloc(conv, dev, calls=50):
    """ccv3d_forward_noalloc on the headline signature: the host time of one
    call (it plans on the host stack every time) and its device time."""
    import torch
    from causal_conv3d_video_b200 import ccv3d

    desc = ccv3d.desc_for(conv)
    plan = ccv3d.Plan(desc)
    dt = torch.bfloat16
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    rnd = lambda shape, sigma: (sigma * torch.randn(shape, generator=gen, device=dev)).to(dt)
    x = rnd((conv.N, conv.T_x, conv.H, conv.W, conv.Cin), 1.0)
    cache = rnd((conv.N, conv.cache_len, conv.H, conv.W, conv.Cin), 1.0)
    w = rnd((conv.Cout, conv.kt, conv.kh, conv.kw, conv.Cin), 1.0 / np.sqrt(conv.Cin * 27))
    b = rnd((conv.Cout,), conv.sigma_b)
    out, nc = plan.alloc_outputs(dev)
    stream = torch.cuda.current_stream(dev)
    f = lambda: ccv3d.ccv3d_forward_noalloc(desc, x, cache, w, b, out, nc, conv.stride,
                                            conv.pad, conv.dilation, stream)
    for _ in range(3):
        f()
    torch.cuda.synchronize()
    host, dev_us = [], []
    for _ in range(calls):
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        t = time.perf_counter()
        f()
        host.append((time.perf_counter() - t) * 1e6)
        eb.record(stream)
        torch.cuda.synchronize()
        dev_us.append(ea.elapsed_time(eb) * 1e3)
    status = ccv3d.ccv3d_noalloc_get_status(stream)
    return {"host_us_per_call_median": round(statistics.median(host), 1),
            "device_us_per_call_median": round(statistics.median(dev_us), 2),
            "status": ccv3d.STATUS.get(status, status),
            "what": "ccv3d_forward_noalloc on the headline signature (persistent kernel, "
                    "scratch in the library's static array): host time of the call, which "
                    "plans on the host stack, and device time"}


def run_quantize(dev, steps=200):
    """The post-decode step: uint8 frames from a decoded 17-frame 720x1280
    RGB fp32 video (47 M values, 235 MB moved per call), timed with CUDA
    events over two rotating buffers (2 x 188 MB > L2); plus the device-to-host
    copy of the frames, fp32 as decoded vs quantised on the device first."""
    import torch
    from causal_conv3d_video_b200 import ccv3d

    shape = (1, 17, 720, 1280, 3)
    n = 1
    for d in shape:
        n *= d
    gen = torch.Generator(device=dev)
    gen.manual_seed(3)
    xs = [torch.rand(shape, generator=gen, device=dev) for _ in range(2)]
    outs = [torch.empty(shape, dtype=torch.uint8, device=dev) for _ in range(2)]
    stream = torch.cuda.current_stream(dev)
    for i in range(6):
        ccv3d.ccv3d_quantize_u8(xs[i % 2], outs[i % 2], stream)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        ccv3d.ccv3d_quantize_u8(xs[i % 2], outs[i % 2], stream)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    us = statistics.median([ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(steps)])
    nbytes = 5 * n
    peaks = load_peaks()
    h32 = torch.empty(shape, dtype=torch.float32, pin_memory=True)
    h8 = torch.empty(shape, dtype=torch.uint8, pin_memory=True)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        best = float("inf")
        for _ in range(3):
            torch.cuda.synchronize()
            ea.record(stream)
            fn()
            eb.record(stream)
            torch.cuda.synchronize()
            best = min(best, ea.elapsed_time(eb))
        return best

    d2h_fp32 = timed(lambda: h32.copy_(xs[0], non_blocking=True))

    def quant_then_copy():
        ccv3d.ccv3d_quantize_u8(xs[0], outs[0], stream)
        h8.copy_(outs[0], non_blocking=True)

    d2h_u8 = timed(quant_then_copy)
    ok = torch.equal(h8.to(dev), outs[0])
    return {"values": n, "us_per_call_median": round(us, 2),
            "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
            "roofline": {"bound": "hbm", "achieved": round(nbytes / (us * 1e-6) / 1e9, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                         "bytes_per_value": 5},
            "d2h_fp32_ms": round(d2h_fp32, 3), "quantize_plus_d2h_u8_ms": round(d2h_u8, 3),
            "copied_back_ok": bool(ok),
            "what": "ccv3d_quantize_u8 on a decoded 17x720x1280x3 fp32 video; D2H into pinned "
                    "host memory of the fp32 video vs quantise-on-device + uint8 copy"}


def run_sequence(args, dev):
    """Time the synthetic 17-frame decode: 164 calls over 28 signatures, each
    module's cache threaded from chunk to chunk (ping-pong buffers), all on one
    stream.  Plans are made once per signature.  Inputs are seeded N(0,1)
    frames generated on the device (timing only; parity is in the tests)."""
    import torch
    from causal_conv3d_video_b200 import ccv3d

    calls = workloads.decode17_schedule()
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    plans, frames, outs, mods = {}, {}, {}, {}
    flops = 0.0
    t_star_us = 0.0  # sum over the calls of max(F/P, B/BW) at the measured peaks
    peaks = load_peaks()
    for call in calls:
        c = call.conv
        sig = workloads.signature(c)
        if sig not in plans:
            plans[sig] = ccv3d.Plan(ccv3d.desc_for(c))
        plan = plans[sig]
        f_i, b_i = algorithmic(c, plan.intervals)
        flops += f_i
        t_star_us += max(f_i / (peaks["bf16_tflops"] * 1e12), b_i / (peaks["hbm_gbs"] * 1e9)) * 1e6
        xs = (1, c.T_x, c.H, c.W, c.Cin)
        if xs not in frames:
            frames[xs] = torch.randn(xs, generator=gen, device=dev).to(torch.bfloat16)
        os_ = plan.out_shape()
        if os_ not in outs:
            outs[os_] = torch.empty(os_, dtype=torch.bfloat16, device=dev)
        if call.module not in mods:
            w = (torch.randn((c.Cout, c.kt, c.kh, c.kw, c.Cin), generator=gen, device=dev)
                 / (c.Cin * c.kt * c.kh * c.kw) ** 0.5).to(torch.bfloat16)
            b = (0.02 * torch.randn((c.Cout,), generator=gen, device=dev)).to(torch.bfloat16)
            cs = (1, 2, c.H, c.W, c.Cin)
            caches = [torch.randn(cs, generator=gen, device=dev).to(torch.bfloat16)
                      for _ in range(2)]
            mods[call.module] = [w, b, caches, 0]
    stream = torch.cuda.current_stream(dev)

    def one_pass(stream=stream):
        for m in mods.values():
            m[3] = 0
        for call in calls:
            c = call.conv
            plan = plans[workloads.signature(c)]
            w, b, caches, cur = mods[call.module]
            cache = caches[cur][:, :c.cache_len] if c.cache_len > 0 else None
            keep = plan.sizes["new_cache_frames"]
            nc = caches[1 - cur][:, :keep]
            plan.forward(frames[(1, c.T_x, c.H, c.W, c.Cin)], cache, w, b,
                         outs[plan.out_shape()], nc, stream)
            mods[call.module][3] = 1 - cur

    for _ in range(2):
        one_pass()
    torch.cuda.synchronize()
    passes = max(1, args.sequence_passes)
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(passes):
        one_pass()
    eb.record(stream)
    torch.cuda.synchronize()
    ms = ea.elapsed_time(eb) / passes
    for plan in plans.values():
        if plan.status() != 0:
            raise RuntimeError("device status after the decode sequence")
    # the same pass captured once as a CUDA graph (164 kernel nodes), replayed
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap):
        one_pass(cap)
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(passes):
        graph.replay()
    eb.record(stream)
    torch.cuda.synchronize()
    ms_graph = ea.elapsed_time(eb) / passes
    for plan in plans.values():
        if plan.status() != 0:
            raise RuntimeError("device status after the graph-replayed decode sequence")
    del graph

    # the same pass with every module's cache in a ring buffer (only the
    # arriving frames of each new cache are written)
    rings = {}
    for call in calls:
        c = call.conv
        m = call.module
        plan = plans[workloads.signature(c)]
        need = c.cache_len + plan.ring_writes()
        if m not in rings or rings[m][1] < need:
            rings[m] = [None, max(need, rings.get(m, [None, 0])[1]), 0]
    for m, r in rings.items():
        c = next(call.conv for call in calls if call.module == m)
        r[0] = torch.randn((1, r[1], c.H, c.W, c.Cin), generator=gen, device=dev).to(torch.bfloat16)

    def ring_pass(stream=stream):
        for call in calls:
            c = call.conv
            plan = plans[workloads.signature(c)]
            w, b = mods[call.module][0], mods[call.module][1]
            ring = rings[call.module]
            ring[2] = plan.forward_ring(frames[(1, c.T_x, c.H, c.W, c.Cin)], ring[0], ring[1],
                                        ring[2], w, b, outs[plan.out_shape()], stream)

    for _ in range(2):
        ring_pass()
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(passes):
        ring_pass()
    eb.record(stream)
    torch.cuda.synchronize()
    ms_ring = ea.elapsed_time(eb) / passes
    graph = torch.cuda.CUDAGraph()
    cap.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap):
        ring_pass(cap)
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    ea.record(stream)
    for _ in range(passes):
        graph.replay()
    eb.record(stream)
    torch.cuda.synchronize()
    ms_ring_graph = ea.elapsed_time(eb) / passes
    for plan in plans.values():
        if plan.status() != 0:
            raise RuntimeError("device status after the ring-buffer decode sequence")
    del graph
    kernels = sorted({p.kernel for p in plans.values()})
    return {"calls": len(calls), "signatures": len(plans), "ms_per_sequence": round(ms, 3),
            "tflops": round(flops / (ms / 1e3) / 1e12, 2), "gflop_per_sequence": round(flops / 1e9, 1),
            "ms_per_sequence_graph": round(ms_graph, 3),
            "tflops_graph": round(flops / (ms_graph / 1e3) / 1e12, 2),
            "ms_per_sequence_ring": round(ms_ring, 3),
            "ms_per_sequence_ring_graph": round(ms_ring_graph, 3),
            "tflops_ring_graph": round(flops / (ms_ring_graph / 1e3) / 1e12, 2),
            "t_star_ms": round(t_star_us / 1e3, 3),
            "frac_of_roofline_graph": round(t_star_us / 1e3 / ms_graph, 4),
            "passes": passes, "kernels": kernels,
            "kernel_per_signature": {f"{k[0]}->{k[1]} k{k[2]}{k[3]}{k[4]} {k[5]}x{k[6]} T{k[7]} C{k[8]}":
                                     p.kernel for k, p in plans.items()},
            "what": "164-call synthetic 17-frame decode, caches threaded, one stream; "
                    "eager launches, and the same pass captured as one CUDA graph; then "
                    "the pass with ring-buffer caches (ccv3d_forward_ring), eager and graph"}


# ------------------------------------------------------------- CPU oracle
class OracleSampler:
    """The FP64 oracle evaluated on random output points of one call: a
    bounded sample of the workload for the CPU baseline."""

    def __init__(self, conv):
        import oracle

        self.oracle = oracle
        self.conv = conv
        self.op = oracle.params(conv.N, conv.Cin, conv.Cout, conv.H, conv.W, conv.T_x,
                                conv.cache_len, kt=conv.kt, kh=conv.kh, kw=conv.kw,
                                pad_t_base=conv.pad_t_base, cache_keep=conv.cache_keep,
                                stride=conv.stride, pad=conv.pad, dilation=conv.dilation,
                                stride_t=conv.stride_t)
        inp = synth.conv_inputs(**conv.synth_kwargs())
        f64 = lambda a: None if a is None else a.astype(np.float64)
        self.x, self.cache, self.w, self.b = (f64(inp["x"]), f64(inp["cache"]),
                                              f64(inp["w"]), f64(inp["bias"]))
        T_o, H_o, W_o, _ = oracle.shape(self.op)
        _, _, o_l, o_h, _ = oracle.tap_scan(self.op)
        self.intervals = {"T_o": T_o, "H_o": H_o, "W_o": W_o, "o_l": o_l, "o_h": o_h}
        self.flops, self.nbytes = algorithmic(conv, self.intervals)
        self.out_shape = (conv.N, T_o, H_o, W_o, conv.Cout)
        self.n_out = int(np.prod(self.out_shape))
        self.cores = oracle.threads()
        self.rng = np.random.default_rng(0)

    def sample(self, n):
        return np.stack([self.rng.integers(0, s, n) for s in self.out_shape], axis=1)

    def run(self, n):
        """Evaluate n random points; returns seconds taken."""
        idx = self.sample(n)
        t = time.perf_counter()
        self.oracle.points(self.op, self.x, self.cache, self.w, self.b, idx)
        return time.perf_counter() - t

    def points_per_s(self):
        self.run(256)
        n = 2048
        return n / max(self.run(n), 1e-6)

    def tflops(self, n, seconds):
        return n * (self.flops / self.n_out) / seconds / 1e12

    def describe(self, n, seconds):
        return (f"{n} random output points of the {self.conv.name} call "
                f"({n / self.n_out:.2%} of its outputs), FP64 direct definition, "
                f"{seconds:.1f} s")


def cpu_baseline(conv, seconds):
    smp = OracleSampler(conv)
    n = int(max(256, min(smp.n_out, smp.points_per_s() * seconds)))
    dt = smp.run(n)
    return {"value": round(smp.tflops(n, dt), 6), "unit": "TFLOP/s", "cores": smp.cores,
            "kind": "oracle", "sample": smp.describe(n, dt),
            "single_thread": _single_thread_baseline(conv, min(4.0, seconds / 3))}


def _single_thread_baseline(conv, seconds):
    """The same oracle on one host core (OpenMP pinned to one thread in a
    child process, since the thread count is fixed when the library loads)."""
    code = ("import json, sys; sys.path.insert(0, sys.argv[1]); import bench; "
            "from causal_conv3d_video_b200 import workloads; "
            "smp = bench.OracleSampler(workloads.WORKLOADS[sys.argv[2]]); "
            "n = int(max(64, min(smp.n_out, smp.points_per_s() * float(sys.argv[3])))); "
            "dt = smp.run(n); "
            "print(json.dumps({'value': round(smp.tflops(n, dt), 6), 'unit': 'TFLOP/s', "
            "'cores': smp.cores, 'sample': smp.describe(n, dt)}))")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code, ROOT, conv.name, str(seconds)], env=env,
                           capture_output=True, text=True, timeout=120 + 4 * seconds)
        return json.loads(r.stdout.strip().splitlines()[-1])
    except Exception as e:  # noqa: BLE001 -- reported in the line
        return {"error": f"{type(e).__name__}: {e}"}


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands, on the host cores."""
    if rank != 0:
        return None
    conv = workloads.WORKLOADS[args.workload]
    smp = OracleSampler(conv)
    rate = smp.points_per_s()
    budget_s = 150.0  # whole warm-up + timed run
    # a step samples at most as many random points as one call has outputs
    n = int(max(16, min(smp.n_out, rate * budget_s / (args.steps + args.warmup))))
    for _ in range(args.warmup):
        smp.run(n)
    t = time.perf_counter()
    for _ in range(args.steps):
        smp.run(n)
    total = time.perf_counter() - t
    value = round(smp.tflops(n * args.steps, total), 6)
    return {
        "impl": "reference",
        "metric": "cached causal Conv3D effective TFLOP/s (bf16), 1 GPU",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": conv.name, "gflop_per_call": round(smp.flops / 1e9, 3),
                   "points_per_step": n},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": smp.cores,
                         "kind": "oracle",
                         "sample": f"{args.steps} steps of " + smp.describe(n, total / args.steps)
                                   + " each"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ccv3d", choices=["ccv3d", "reference"])
    ap.add_argument("--workload", default=workloads.BENCH_WORKLOAD.name,
                    choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sequence", action="store_true",
                    help="skip the 164-call synthetic decode sequence leg")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload legs")
    ap.add_argument("--ring", action="store_true",
                    help="time the headline workload with a ring-buffer cache "
                         "(ccv3d_forward_ring) instead of ping-pong new_cache buffers")
    ap.add_argument("--sequence-passes", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        line = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
