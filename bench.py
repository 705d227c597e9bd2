#!/usr/bin/env python
"""Benchmark of the low-bit quantized linear layer library on B200.

Headline workload (one "step"): the seven linear layers of one LLaMA-3-8B
transformer block (q, k, v, o: 4096/1024 x 4096; gate, up: 14336 x 4096;
down: 4096 x 14336), frozen weights quantized with the group-wise MinMax
quantizer to INT4 with group 128, forward dequantize-GEMM at decode sizes
M = 1 and M = 16 tokens.  Seven independently drawn copies of the weight set
rotate from pass to pass, so every pass streams weights that are not in L2.
Metric: weight GB/s (algorithmic bytes: packed codes + fp16 scales/zeros + X
+ Y, per call) over the whole step, and the dominant kernel's fraction of the
measured HBM bandwidth.

`--impl reference` times the CPU oracle on a bounded sample of the same
workload (the oracle is the reference implementation of this project).

Runs under torchrun for N > 1 as independent replicas (the workload does not
shard; nothing crosses GPUs on the data path): barrier + max-over-ranks
timing, value = all ranks' units / that time.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dequant-GEMM TFLOP/s & weight GB/s at 8B/70B layer shapes, M=1..4096; % roofline"
DECODE_M = (1, 16)
COPIES = 7


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=700)
    ap.add_argument("--warmup", type=int, default=14)
    ap.add_argument("--impl", choices=["lbq", "reference"], default="lbq")
    ap.add_argument("--rows", choices=["all", "none"], default="all",
                    help="also measure the other workloads (training step, 70B codebook, mixed, quantize)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="run one kernel configuration `reps` times and exit (for ncu captures): "
                         "decode_<matrix>_m<M> | layerset_8b_m<M> | train_<matrix>_{fwd,bwd,grads} | "
                         "traingrp_gateup_{fwd,bwd} | "
                         "codebook70b_<matrix>_m<M> | quantize_<matrix>_{int4,codebook} | merge_<matrix>_r16 | "
                         "select_<matrix>_q")
    ap.add_argument("--reps", type=int, default=3)
    return ap.parse_args()


# ----------------------------------------------------------------------------- peaks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# The sources that decide what the decode GEMV kernel does and how it is
# launched: the kernel, the headers it includes and its host-side plan.
GEMV_SOURCES = ("common.cuh", "dqgemm.cuh", "dqgemv.cuh", "dqgemv_host.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "qlora_quantized_linear_b200", "csrc")
    for f in GEMV_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampled every 50 ms in the background; each line is stamped
    with the host time it was read, so a time window can be selected."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.samples = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        win = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(p[0]) for p in win if p[0].replace(".", "").isdigit()]
        smax = [float(p[1]) for p in win if p[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in win for i in range(4) if p[4 + i].lower() == "active"})
        power = [float(p[2]) for p in win if p[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(win), "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- distributed plumbing
class Dist:
    """One process per GPU (torchrun env).  NCCL on GPUs; gloo when there is
    no GPU (or LBQ_DIST_BACKEND=gloo), which the CPU tests use."""

    def __init__(self):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.torch = torch
        self.backend = os.environ.get("LBQ_DIST_BACKEND") or ("nccl" if torch.cuda.is_available() else "gloo")
        if self.world > 1:
            import datetime
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                                     device_id=torch.device("cuda", self.local))
            else:
                torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)

    def barrier(self):
        if self.world > 1:
            self.torch.distributed.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return x
        dev = "cuda" if self.backend == "nccl" else "cpu"
        t = self.torch.tensor([x], dtype=self.torch.float64, device=dev)
        self.torch.distributed.all_reduce(t, op=self.torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.torch.distributed.destroy_process_group()


def replica_value(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput of N independent replicas (weak scaling): the
    units all ranks processed over the slowest rank's device time, in G/s."""
    return units_per_rank * world / (ms_max / 1e3) / 1e9


# ----------------------------------------------------------------------------- byte / flop accounting
def gemm_bytes(m, n, k, bits=4, group=128, rank=0, codebook=False, dq=False):
    """Algorithmic bytes of one forward call: packed codes + per-group
    metadata + X (bf16) + Y (fp32) (+ adapter A, B, T)."""
    w = n * k * bits // 8
    if codebook:
        nb = n * k // 64
        meta = nb + 4 * ((nb + 255) // 256) + 4 if dq else 4 * nb
    else:
        meta = 4 * (n * k // group)
    b = w + meta + 2 * m * k + 4 * m * n
    if rank:
        b += 2 * rank * (k + n) + 4 * m * rank
    return b


def gemm_flops(m, n, k, rank=0):
    return 2 * m * n * k + (2 * m * rank * (k + n) if rank else 0)


# ----------------------------------------------------------------------------- the decode workload
class Decode8B:
    """The decode step: the seven layers at M = 1 and at M = 16, each size one
    grouped forward call (one launch of the decode GEMV over the seven
    weights), each size on its own rotating weight copy."""

    def __init__(self, lbq, syn, torch):
        import ctypes
        self.lbq, self.torch = lbq, torch
        self.shapes = syn.LLAMA3_8B_SHAPES
        dev = "cuda"
        self.qw = []
        for c in range(COPIES):
            layer = {}
            for i, (name, (n, k)) in enumerate(self.shapes.items()):
                W = syn.weight_bf16(n, k, 0.02, seed=100 * c + i, outlier_frac=0.001, outlier_scale=20.0, device=dev)
                layer[name] = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W)
                del W
            self.qw.append(layer)
        self.X = {(m, k): syn.normal_bf16((m, k), 1.0, seed=7 * m + k, device=dev) for m in DECODE_M
                  for k in {kk for (_, kk) in self.shapes.values()}}
        self.Y = {(m, name): torch.empty((m, n), dtype=torch.float32, device=dev)
                  for m in DECODE_M for name, (n, _) in self.shapes.items()}
        self.calls_per_step = len(DECODE_M)                  # grouped launches per step
        self.step_bytes = sum(gemm_bytes(m, n, k) for m in DECODE_M for (n, k) in self.shapes.values())
        # the C arguments of every (size, copy): one lbq_fwd_problem array each
        self.problems = {}
        for m in DECODE_M:
            for c in range(COPIES):
                arr = (lbq.lbq_fwd_problem * len(self.shapes))()
                for i, (name, (n, k)) in enumerate(self.shapes.items()):
                    arr[i] = lbq.lbq_fwd_problem(X=self.X[(m, k)].data_ptr(), q=ctypes.pointer(self.qw[c][name].struct),
                                                 A=None, B=None, rank=0, s=0.0, Y=self.Y[(m, name)].data_ptr(),
                                                 T_save=None)
                self.problems[(m, c)] = arr
        self.ws_bytes = max(lbq.lbq_linear_fwd_grouped_workspace_size(m, self.problems[(m, 0)], len(self.shapes))
                            for m in DECODE_M)
        self.ws = lbq._workspace(self.ws_bytes, dev)
        self.ws_single = {(m, name): lbq._workspace(self._ws_size(m, self.qw[0][name]), dev)
                          for m in DECODE_M for name in self.shapes}
        torch.cuda.synchronize()

    def _ws_size(self, m, q):
        import ctypes
        return self.lbq.lbq_linear_fwd_workspace_size(m, ctypes.byref(q.struct), 0)

    def call_group(self, m, copy, stream_handle):
        rc = self.lbq.lbq_linear_fwd_grouped(m, self.problems[(m, copy)], len(self.shapes), self.ws.data_ptr(),
                                             self.ws_bytes, stream_handle)
        if rc != 0:
            raise RuntimeError(f"lbq_linear_fwd_grouped returned {rc}")

    def call(self, m, name, copy, stream=None):
        k = self.shapes[name][1]
        self.lbq.linear_fwd(self.X[(m, k)], self.qw[copy][name], Y=self.Y[(m, name)],
                            workspace=self.ws_single[(m, name)], stream=stream)

    def capture(self, phase: int, stream, probe: bool = False):
        """CUDA graph of one step: both decode sizes, each one grouped launch
        over the layer set on its own weight copy (back to back; each may
        overlap the tail of the one before it).  The probe graphs instead make
        the 14 per-matrix calls with timing events around every call, which
        serialises them, to give per-matrix durations."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        evs = []
        with torch.cuda.graph(g, stream=stream):
            for j, m in enumerate(DECODE_M):
                copy = (2 * phase + j) % COPIES
                if not probe:
                    self.call_group(m, copy, stream.cuda_stream)
                    continue
                for name in self.shapes:
                    e0 = torch.cuda.Event(enable_timing=True, external=True)
                    e1 = torch.cuda.Event(enable_timing=True, external=True)
                    e0.record()
                    self.call(m, name, copy)
                    e1.record()
                    evs.append((m, name, e0, e1))
        return g, evs


def run_decode(args, dist, lbq, syn, torch, peaks):
    wl = Decode8B(lbq, syn, torch)
    stream = torch.cuda.Stream()
    # eager warm-up (module loading, function attributes), then capture
    with torch.cuda.stream(stream):
        for c in range(2):
            for m in DECODE_M:
                wl.call_group(m, c, stream.cuda_stream)
                for name in wl.shapes:
                    wl.call(m, name, c)
    torch.cuda.synchronize()
    graphs = [wl.capture(ph, stream) for ph in range(COPIES)]
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    time.sleep(0.3)
    for i in range(args.warmup):
        graphs[i % COPIES][0].replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    host0 = time.time()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            graphs[(args.warmup + i) % COPIES][0].replay()
        t_end.record(stream)
    torch.cuda.synchronize()
    host1 = time.time()
    dist.barrier()
    ms = t_start.elapsed_time(t_end)
    # keep the GPU busy a little longer when the timed region is too short for
    # the 50 ms clock sampler, with the same graphs on the same stream
    ext_until = host1
    if host1 - host0 < 1.0:
        with torch.cuda.stream(stream):
            t_ext = time.time()
            i = 0
            while time.time() - t_ext < 1.0:
                for _ in range(50):
                    graphs[i % COPIES][0].replay()
                    i += 1
                torch.cuda.synchronize()
        ext_until = time.time()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(host0, ext_until)
    clocks["window_s"] = round(ext_until - host0, 3)
    clocks["timed_s"] = round(host1 - host0, 3)

    ms_max = dist.max(ms)
    value = replica_value(args.steps * wl.step_bytes, dist.world, ms_max)

    # The timed region launches nothing but the dominant kernel (the grouped
    # decode GEMV, one launch per decode size), back to back: its average
    # launch duration is the region's device time over the launches in it.
    launches = args.steps * wl.calls_per_step
    avg_launch_ms = ms / launches
    per_launch_bytes = wl.step_bytes / wl.calls_per_step
    achieved = per_launch_bytes / (avg_launch_ms / 1e3) / 1e9
    traffic = profiled_traffic("dqgemv_decode_8b")
    roofline = {"kernel": "dqgemv_grouped_kernel (one launch per decode size over the 7-matrix layer set)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": peaks["source"], "traffic": traffic,
                "per_launch_bytes_avg": int(per_launch_bytes), "avg_launch_us": round(1e3 * avg_launch_ms, 3),
                "launches_timed": launches}

    # per-size launch durations (one grouped launch between events) and
    # per-matrix durations (single calls between events), after the timed region
    per_size = {}
    for m in DECODE_M:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 50
        with torch.cuda.stream(stream):
            e0.record(stream)
            for r in range(reps):
                wl.call_group(m, r % COPIES, stream.cuda_stream)
            e1.record(stream)
        torch.cuda.synchronize()
        us = 1e3 * e0.elapsed_time(e1) / reps
        b = sum(gemm_bytes(m, n, k) for (n, k) in wl.shapes.values())
        per_size[f"M{m}"] = {"us": round(us, 2), "GB/s": round(b / us / 1e3, 1)}
    probes = [wl.capture(ph, stream, probe=True) for ph in range(COPIES)]
    with torch.cuda.stream(stream):
        for _ in range(2):
            for g, _evs in probes:
                g.replay()
    torch.cuda.synchronize()
    per = {}
    for g, evs in probes:
        for (m, name, e0, e1) in evs:
            per.setdefault((m, name), []).append(e0.elapsed_time(e1))
    per_matrix = {f"M{m}/{name}": {"us": round(1e3 * statistics.median(v), 2),
                                     "GB/s": round(gemm_bytes(m, *wl.shapes[name]) / (statistics.median(v) / 1e3) / 1e9, 1)}
                  for (m, name), v in per.items()}
    per_matrix["grouped_launch"] = per_size
    del probes

    # end to end through the public API: pinned host X in, Y out, every call
    e2e = run_decode_e2e(args, dist, wl, lbq, torch, stream)
    del graphs
    return wl, value, ms_max, clocks, roofline, per_matrix, e2e


def run_decode_e2e(args, dist, wl, lbq, torch, stream):
    """The decode step end to end through the C ABI, as a serving loop runs
    it: every step copies that step's activations from pinned host memory to
    the device (one copy of the four distinct X of the layer set), makes the
    two grouped forward calls (seven layers each) and reads all 14 outputs
    back to pinned host memory (one copy).  The copies run on their own
    streams (host to device, device to host) with the host and device buffers
    doubled, so step i's outputs travel back and step i + 1's inputs travel
    in while step i + 1 (or i) computes; events order each buffer's reuse.
    Wall clock from the host, synchronised at both ends, between barriers;
    with several ranks, the units of all ranks over the slowest rank's
    time."""
    import ctypes
    xkeys = sorted(wl.X)                                      # (m, k): the distinct activations
    ykeys = [(m, name) for m in DECODE_M for name in wl.shapes]
    xn = {key: wl.X[key].numel() for key in xkeys}
    yn = {key: wl.Y[key].numel() for key in ykeys}
    nb = 2                                                    # buffers in flight
    xh = [torch.empty(sum(xn.values()), dtype=torch.bfloat16).pin_memory() for _ in range(nb)]
    yh = [torch.empty(sum(yn.values()), dtype=torch.float32).pin_memory() for _ in range(nb)]
    xd = [torch.empty_like(xh[0], device="cuda") for _ in range(nb)]
    yd = [torch.empty_like(yh[0], device="cuda") for _ in range(nb)]
    xview = [{} for _ in range(nb)]
    yview = [{} for _ in range(nb)]
    for b in range(nb):
        off = 0
        for key in xkeys:                                     # host copy of the inputs, views on the device
            xh[b][off:off + xn[key]].copy_(wl.X[key].reshape(-1).cpu())
            xview[b][key] = xd[b][off:off + xn[key]]
            off += xn[key]
        off = 0
        for key in ykeys:
            yview[b][key] = yd[b][off:off + yn[key]]
            off += yn[key]
    sh = stream.cuda_stream
    calls = []                                                # [phase][buffer]: one grouped call per decode size
    for phase in range(COPIES):
        per_buf = []
        for b in range(nb):
            row = []
            for j, m in enumerate(DECODE_M):
                copy = (2 * phase + j) % COPIES
                arr = (lbq.lbq_fwd_problem * len(wl.shapes))()
                for i, (name, (n, k)) in enumerate(wl.shapes.items()):
                    arr[i] = lbq.lbq_fwd_problem(X=xview[b][(m, k)].data_ptr(),
                                                 q=ctypes.pointer(wl.qw[copy][name].struct), A=None, B=None, rank=0,
                                                 s=0.0, Y=yview[b][(m, name)].data_ptr(), T_save=None)
                row.append((m, arr, len(wl.shapes), wl.ws.data_ptr(), wl.ws_bytes, sh))
            per_buf.append(row)
        calls.append(per_buf)
    fwd = lbq.lbq_linear_fwd_grouped
    h2d = xh[0].numel() * xh[0].element_size()
    d2h = yh[0].numel() * yh[0].element_size()
    steps = max(3, min(args.steps, 50))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    x_ready = [torch.cuda.Event() for _ in range(nb)]         # inputs of buffer b on the device
    y_ready = [torch.cuda.Event() for _ in range(nb)]         # outputs of buffer b written (inputs read)
    y_read = [torch.cuda.Event() for _ in range(nb)]          # outputs of buffer b copied to the host

    def one_step(i):
        b = i % nb
        with torch.cuda.stream(s_in):
            s_in.wait_event(y_ready[b])                       # step i - nb has read these inputs
            xd[b].copy_(xh[b], non_blocking=True)
            x_ready[b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(x_ready[b])
            stream.wait_event(y_read[b])                      # step i - nb's outputs are on the host
            for a in calls[i % COPIES][b]:
                rc = fwd(*a)
                if rc != 0:
                    raise RuntimeError(f"lbq_linear_fwd_grouped returned {rc}")
            y_ready[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(y_ready[b])
            yh[b].copy_(yd[b], non_blocking=True)
            y_read[b].record(s_out)

    for i in range(3):
        one_step(i)
    torch.cuda.synchronize()
    dist.barrier()
    t0 = time.perf_counter()
    for i in range(steps):
        one_step(i)
    torch.cuda.synchronize()                                  # every step's outputs are on the host
    dt = time.perf_counter() - t0
    dist.barrier()
    dt_max = dist.max(dt)
    return {"value": round(replica_value(steps * wl.step_bytes, dist.world, 1e3 * dt_max), 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "lbq_linear_fwd_grouped through the C ABI, one call per decode size (7 layers each); per step "
                    "and rank one pinned host->device copy of the four distinct activations and one device->host "
                    "copy of the 14 outputs, on their own streams with double buffers, overlapping the "
                    "neighbouring steps' calls"}


# ----------------------------------------------------------------------------- extra rows
def time_graph(torch, fn, stream, reps=5, warm=2):
    """Capture fn() once and time `reps` replays with CUDA events; returns ms per replay."""
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def row_training(lbq, syn, torch, peaks, stream):
    """QLoRA training step on the 8B MLP shapes at M = 4096, rank 16, INT4 g128."""
    m, r, s = 4096, 16, 2.0
    out = {}
    tot_flops = tot_ms = 0.0
    keep, per = {}, {}
    for i, name in enumerate(("gate", "up", "down")):
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=500 + i, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W)
        del W
        X = syn.normal_bf16((m, k), 1.0, seed=600 + i, device="cuda")
        A = syn.normal_bf16((r, k), 0.01, seed=700 + i, device="cuda")
        B = syn.normal_bf16((n, r), 0.01, seed=800 + i, device="cuda")
        dY = syn.normal_bf16((m, n), 0.1, seed=900 + i, device="cuda")
        Y = torch.empty((m, n), dtype=torch.float32, device="cuda")
        T = torch.empty((m, r), dtype=torch.float32, device="cuda")
        dX = torch.empty((m, k), dtype=torch.float32, device="cuda")
        U = torch.empty((m, r), dtype=torch.float32, device="cuda")
        dA = torch.empty((r, k), dtype=torch.float32, device="cuda")
        dB = torch.empty((n, r), dtype=torch.float32, device="cuda")
        f_ms = time_graph(torch, lambda: lbq.linear_fwd(X, qw, A, B, s, Y=Y, T=T, stream=stream), stream)
        b_ms = time_graph(torch, lambda: lbq.linear_bwd(dY, qw, A, B, s, dX=dX, U=U, stream=stream), stream)
        g_ms = time_graph(torch, lambda: lbq.lora_grads(X, dY, T, U, s, dA=dA, dB=dB, stream=stream), stream)
        f_fl = gemm_flops(m, n, k, r)
        b_fl = gemm_flops(m, n, k, r)
        g_fl = 4 * m * r * (n + k) // 2
        out[name] = {"fwd_ms": round(f_ms, 3), "fwd_TFLOP/s": round(f_fl / f_ms / 1e9, 1),
                     "bwd_ms": round(b_ms, 3), "bwd_TFLOP/s": round(b_fl / b_ms / 1e9, 1),
                     "grads_ms": round(g_ms, 3),
                     "fwd_frac_of_bf16_peak": round(f_fl / f_ms / 1e9 / peaks["bf16_tflops"], 3),
                     "bwd_frac_of_bf16_peak": round(b_fl / b_ms / 1e9 / peaks["bf16_tflops"], 3)}
        tot_flops += f_fl + b_fl + g_fl
        tot_ms += f_ms + b_ms + g_ms
        per[name] = (f_ms, b_ms, g_ms, f_fl)
        if name != "down":
            keep[name] = (qw, X, A, B, dY)
        del qw, X, A, B, dY, Y, T, dX, U, dA, dB
        torch.cuda.empty_cache()
    out["step_TFLOP/s"] = round(tot_flops / tot_ms / 1e9, 1)
    out["step_ms"] = round(tot_ms, 3)
    # gate and up (the same shape) as one grouped launch for the forward and
    # one for the backward, as an MLP block runs them
    fwd_probs = [(keep[nm][1], keep[nm][0], keep[nm][2], keep[nm][3], s) for nm in ("gate", "up")]
    bwd_probs = [(keep[nm][4], keep[nm][0], keep[nm][2], keep[nm][3], s) for nm in ("gate", "up")]
    gf_ms = time_graph(torch, lambda: lbq.linear_fwd_grouped(fwd_probs, stream=stream), stream)
    gb_ms = time_graph(torch, lambda: lbq.linear_bwd_grouped(bwd_probs, stream=stream), stream)
    fl2 = per["gate"][3] + per["up"][3]
    out["gate_up_grouped"] = {"fwd_ms": round(gf_ms, 3), "fwd_TFLOP/s": round(fl2 / gf_ms / 1e9, 1),
                              "fwd_frac_of_bf16_peak": round(fl2 / gf_ms / 1e9 / peaks["bf16_tflops"], 3),
                              "bwd_ms": round(gb_ms, 3), "bwd_TFLOP/s": round(fl2 / gb_ms / 1e9, 1),
                              "bwd_frac_of_bf16_peak": round(fl2 / gb_ms / 1e9 / peaks["bf16_tflops"], 3)}
    step_g = gf_ms + gb_ms + per["down"][0] + per["down"][1] + sum(per[nm][2] for nm in per)
    out["step_grouped_ms"] = round(step_g, 3)
    out["step_grouped_TFLOP/s"] = round(tot_flops / step_g / 1e9, 1)
    out["peak_bf16_tflops"] = peaks["bf16_tflops"]
    del keep, fwd_probs, bwd_probs
    torch.cuda.empty_cache()
    return out


def row_codebook70b(lbq, syn, torch, peaks, stream):
    cb = syn.codebook_normal16()
    out = {}
    for i, (name, (n, k)) in enumerate(syn.LLAMA3_70B_SHAPES.items()):
        W = syn.weight_bf16(n, k, 0.015, seed=1000 + i, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=True, codebook=cb)
        q_ms = time_graph(torch, lambda: qw.quantize(W, stream=stream), stream, reps=5)
        del W
        nb = n * k // 64
        q_bytes = 2 * n * k + n * k // 2 + 4 * nb + nb + 4 * ((nb + 255) // 256)
        row = {"quantize_us": round(1e3 * q_ms, 1), "quantize_GB/s": round(q_bytes / q_ms / 1e6, 1),
               "quantize_frac_hbm": round(q_bytes / q_ms / 1e6 / peaks["hbm_gbs"], 3)}
        for m in (1, 2048):
            X = syn.normal_bf16((m, k), 1.0, seed=1100 + m, device="cuda")
            Y = torch.empty((m, n), dtype=torch.float32, device="cuda")
            ws = lbq._workspace(lbq.lbq_linear_fwd_workspace_size(m, lbq.ctypes.byref(qw.struct), 0), "cuda")
            ms = time_graph(torch, lambda: lbq.linear_fwd(X, qw, Y=Y, workspace=ws, stream=stream), stream,
                            reps=10 if m == 1 else 3)
            b = gemm_bytes(m, n, k, codebook=True, dq=True)
            fl = gemm_flops(m, n, k)
            row[f"M{m}_us"] = round(1e3 * ms, 1)
            row[f"M{m}_GB/s"] = round(b / ms / 1e6, 1)
            row[f"M{m}_TFLOP/s"] = round(fl / ms / 1e9, 1)
            row[f"M{m}_roofline_frac"] = round(max(b / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
                                               / (ms / 1e3), 3)
            del X, Y, ws
        out[f"{name} {n}x{k}"] = row
        del qw
        torch.cuda.empty_cache()
    return out


def row_mixed(lbq, syn, torch, peaks, stream):
    shapes = syn.LLAMA3_8B_SHAPES
    bits = syn.layer_mix_choice(seed=0)
    out = {"layer_mix_bits": bits}
    layer = {}
    mixw = {}
    for i, (name, (n, k)) in enumerate(shapes.items()):
        W = syn.weight_bf16(n, k, 0.02, seed=1200 + i, outlier_frac=0.001, device="cuda")
        layer[name] = lbq.QuantizedWeight(n, k, "minmax", bits[name]).quantize(W)
        perm, n4 = syn.channel_mix_perm(n, 0.25, seed=i)
        Wp = W[torch.from_numpy(perm.astype("int64")).cuda()]
        hi = lbq.QuantizedWeight(n4, k, "minmax", 4).quantize(Wp[:n4].contiguous())
        lo = lbq.QuantizedWeight(n - n4, k, "minmax", 2).quantize(Wp[n4:].contiguous())
        mixw[name] = lbq.ChannelMixWeight(hi, lo, perm)
        del W, Wp
    import ctypes
    for m in (16, 512):
        Xs = {k: syn.normal_bf16((m, k), 1.0, seed=1300 + k, device="cuda") for k in (4096, 14336)}
        Ys = {name: torch.empty((m, n), dtype=torch.float32, device="cuda") for name, (n, _) in shapes.items()}
        # layer-mix: the seven layers in one grouped call (one launch at M = 16)
        probs = (lbq.lbq_fwd_problem * len(shapes))()
        for i, (nm, (n, k)) in enumerate(shapes.items()):
            probs[i] = lbq.lbq_fwd_problem(X=Xs[k].data_ptr(), q=ctypes.pointer(layer[nm].struct), A=None, B=None,
                                           rank=0, s=0.0, Y=Ys[nm].data_ptr(), T_save=None)
        gws_bytes = lbq.lbq_linear_fwd_grouped_workspace_size(m, probs, len(shapes))
        gws = lbq._workspace(gws_bytes, "cuda")

        def layer_mix_step():
            rc = lbq.lbq_linear_fwd_grouped(m, probs, len(shapes), None if gws is None else gws.data_ptr(), gws_bytes,
                                            stream.cuda_stream)
            if rc != 0:
                raise RuntimeError(f"lbq_linear_fwd_grouped returned {rc}")

        # channel-mix: the seven layers' halves in one grouped call (two
        # launches of the decode GEMV at M = 16; one GEMM per half at M = 512)
        mprobs = (lbq.lbq_mix_problem * len(shapes))()
        for i, (nm, (n, k)) in enumerate(shapes.items()):
            mprobs[i] = lbq.lbq_mix_problem(X=Xs[k].data_ptr(), q=ctypes.pointer(mixw[nm].struct), A=None, B=None,
                                            rank=0, s=0.0, Y=Ys[nm].data_ptr(), T_save=None)
        mws_bytes = lbq.lbq_linear_fwd_mix_grouped_workspace_size(m, mprobs, len(shapes))
        mws = lbq._workspace(mws_bytes, "cuda")

        def channel_mix_step():
            rc = lbq.lbq_linear_fwd_mix_grouped(m, mprobs, len(shapes), None if mws is None else mws.data_ptr(),
                                                mws_bytes, stream.cuda_stream)
            if rc != 0:
                raise RuntimeError(f"lbq_linear_fwd_mix_grouped returned {rc}")
        for label, step, bytes_of in (
                ("layer_mix", layer_mix_step,
                 lambda nm, n, k: gemm_bytes(m, n, k, bits=bits[nm], group=128 if bits[nm] == 4 else 64)),
                ("channel_mix", channel_mix_step,
                 lambda nm, n, k: gemm_bytes(m, mixw[nm].hi.n, k) + gemm_bytes(m, mixw[nm].lo.n, k, bits=2, group=64)
                 - 2 * m * k)):
            ms = time_graph(torch, step, stream, reps=10)
            b = sum(bytes_of(nm, n, k) for nm, (n, k) in shapes.items())
            fl = sum(gemm_flops(m, n, k) for (n, k) in shapes.values())
            out[f"{label}_M{m}"] = {"us": round(1e3 * ms, 1), "GB/s": round(b / ms / 1e6, 1),
                                     "TFLOP/s": round(fl / ms / 1e9, 2),
                                     "roofline_frac": round(max(b / (peaks["hbm_gbs"] * 1e9),
                                                                fl / (peaks["bf16_tflops"] * 1e12)) / (ms / 1e3), 3)}
    return out


def row_quantize8b(lbq, syn, torch, peaks, stream):
    out = {}
    tot_b = tot_ms = 0.0
    for i, (name, (n, k)) in enumerate(syn.LLAMA3_8B_SHAPES.items()):
        W = syn.weight_bf16(n, k, 0.02, seed=1400 + i, outlier_frac=0.001, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4)
        ms = time_graph(torch, lambda: qw.quantize(W, stream=stream), stream, reps=10)
        b = 2 * n * k + n * k // 2 + 4 * (n * k // 128)
        tot_b += b
        tot_ms += ms
        del W, qw
    out["int4_g128_layer_set_GB/s"] = round(tot_b / tot_ms / 1e6, 1)
    out["int4_g128_layer_set_us"] = round(1e3 * tot_ms, 1)
    out["frac_hbm"] = round(tot_b / tot_ms / 1e6 / peaks["hbm_gbs"], 3)
    return out


def row_merge8b(lbq, syn, torch, peaks, stream):
    """Merging a rank-16 adapter into each 8B MLP matrix (INT4 g128 -> bf16),
    then re-quantizing the merged weight; algorithmic bytes: packed weight and
    constants + A + B read, bf16 written (merge); bf16 read, packed weight and
    constants written (re-quantize)."""
    out = {}
    r = 16
    for i, name in enumerate(("gate", "down")):
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=1500 + i, outlier_frac=0.001, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W, stream=stream)
        A = syn.normal_bf16((r, k), 0.01, seed=1510 + i, device="cuda")
        B = syn.normal_bf16((n, r), 0.01, seed=1520 + i, device="cuda")
        merged = torch.empty((n, k), dtype=torch.bfloat16, device="cuda")
        q2 = lbq.QuantizedWeight(n, k, "minmax", 4)
        ms_m = time_graph(torch, lambda: lbq.merge_lora(qw, A, B, 2.0, out=merged, stream=stream), stream, reps=10)
        ms_q = time_graph(torch, lambda: q2.quantize(merged, stream=stream), stream, reps=10)
        packed = n * k // 2 + 4 * (n * k // 128)
        b_m = packed + 2 * r * (n + k) + 2 * n * k
        b_q = 2 * n * k + packed
        out[f"{name} {n}x{k}"] = {"merge_us": round(1e3 * ms_m, 1), "merge_GB/s": round(b_m / ms_m / 1e6, 1),
                                  "merge_frac_hbm": round(b_m / ms_m / 1e6 / peaks["hbm_gbs"], 3),
                                  "requantize_us": round(1e3 * ms_q, 1),
                                  "requantize_GB/s": round(b_q / ms_q / 1e6, 1)}
        del W, qw, A, B, merged, q2
    return out


def row_channel_select(lbq, syn, torch, peaks, stream):
    """Choosing the INT4 quarter of each 8B MLP matrix's output channels by
    sensitivity (lbq_channel_mix_select, 128 calibration tokens); algorithmic
    bytes: the bf16 weight and the calibration activations read, the
    permutation written."""
    out = {}
    t = 128
    for i, name in enumerate(("gate", "down")):
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=1600 + i, outlier_frac=0.001, device="cuda")
        X = syn.normal_bf16((t, k), 1.0, seed=1610 + i, device="cuda")
        n4 = n // 4
        perm = torch.empty(n, dtype=torch.int32, device="cuda")
        nws = lbq.lbq_channel_mix_select_workspace_size(n, k)
        ws = torch.empty(nws, dtype=torch.uint8, device="cuda")

        def fn():
            rc = lbq.lbq_channel_mix_select(W.data_ptr(), n, k, X.data_ptr(), t, n4, None, perm.data_ptr(),
                                            ws.data_ptr(), nws, stream.cuda_stream)
            if rc != 0:
                raise RuntimeError(f"lbq_channel_mix_select returned {rc}")
        ms = time_graph(torch, fn, stream, reps=10)
        b = 2 * n * k + 2 * t * k + 4 * n
        out[f"{name} {n}x{k}"] = {"us": round(1e3 * ms, 1), "GB/s": round(b / ms / 1e6, 1),
                                  "frac_hbm": round(b / ms / 1e6 / peaks["hbm_gbs"], 3)}
        del W, X
    return out


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(rows: int, threads: int = 0):
    """The oracle's forward on `rows` output rows of the gate matrix (K = 4096)
    at M = 1 and M = 16; returns (bytes, seconds, threads used)."""
    import numpy as np
    import oracle
    from qlora_quantized_linear_b200 import synthetic as syn
    if threads:
        oracle.set_threads(threads)
    n, k = syn.LLAMA3_8B_SHAPES["gate"]
    W = syn.weight_bf16(rows, k, 0.02, seed=0, outlier_frac=0.001)
    codes, scale, zero = oracle.minmax_quantize(syn.bits_u16(W), 4, 128)
    packed = oracle.pack(codes, 4)
    total_b, total_s = 0, 0.0
    for m in DECODE_M:
        X = syn.bits_u16(syn.normal_bf16((m, k), 1.0, seed=7 * m + k))
        ri = np.repeat(np.arange(m), rows)
        ci = np.tile(np.arange(rows), m)
        t0 = time.perf_counter()
        oracle.linear_fwd_sampled_minmax(X, packed, scale, zero, rows, k, 4, 128, ri, ci)
        total_s += time.perf_counter() - t0
        total_b += gemm_bytes(m, rows, k)
    return total_b, total_s, oracle.get_threads()


def cpu_baseline():
    """The oracle on whole gate matrices (14336 x 4096) at M = 1 and M = 16,
    repeated until about 10 s of CPU time has been spent."""
    rows = 14336
    tb = ts = 0.0
    reps = 0
    thr = 1
    while ts < 10.0 and reps < 20:
        b, s, thr = oracle_sample(rows)
        tb += b
        ts += s
        reps += 1
    return {"value": round(tb / ts / 1e9, 4), "unit": "GB/s", "cores": thr, "kind": "oracle",
            "host_cpus": os.cpu_count(),
            "sample": f"{reps} x gate 14336x4096 INT4 g128 at M=1 and M=16 "
                      f"({tb / 1e6:.0f} MB of algorithmic traffic in {ts:.1f} s)"}


def run_reference(args):
    """--impl reference: the CPU oracle on a bounded sample per step."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    rows = 512
    for _ in range(args.warmup):
        oracle_sample(rows)
    tb = ts = 0.0
    thr = 1
    for _ in range(args.steps):
        b, s, thr = oracle_sample(rows)
        tb += b
        ts += s
    value = round(tb / ts / 1e9, 4)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * ts / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "LLaMA-3-8B layer set INT4 g128 decode (oracle sample: gate rows at M=1,16)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": thr, "kind": "oracle",
                             "sample": f"gate 14336x4096 INT4 g128, first {rows} output rows, M=1 and M=16 per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- single cases (ncu)
def run_case(args):
    """One kernel configuration, `reps` times, on fresh inputs; prints the
    CUDA-event time of the last call.  Inputs of the 8B/70B shapes exceed no
    more than a few hundred MB on the device."""
    import torch
    from qlora_quantized_linear_b200 import lbq, synthetic as syn
    torch.cuda.set_device(0)
    kind, rest = args.case.split("_", 1)
    name, arg = rest.rsplit("_", 1)
    stream = torch.cuda.current_stream()
    if kind == "layerset":
        # the 8B layer set in one grouped forward call at M = int(arg[1:])
        import ctypes
        m = int(arg[1:])
        qws, Xs = [], {}
        for i, (nm, (n, k)) in enumerate(syn.LLAMA3_8B_SHAPES.items()):
            W = syn.weight_bf16(n, k, 0.02, seed=10 + i, outlier_frac=0.001, device="cuda")
            qws.append(lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W))
            del W
            if k not in Xs:
                Xs[k] = syn.normal_bf16((m, k), 1.0, seed=2 + k, device="cuda")
        Ys = [torch.empty((m, q.n), dtype=torch.float32, device="cuda") for q in qws]
        probs = (lbq.lbq_fwd_problem * len(qws))()
        for i, q in enumerate(qws):
            probs[i] = lbq.lbq_fwd_problem(X=Xs[q.k].data_ptr(), q=ctypes.pointer(q.struct), A=None, B=None, rank=0,
                                           s=0.0, Y=Ys[i].data_ptr(), T_save=None)
        nws = lbq.lbq_linear_fwd_grouped_workspace_size(m, probs, len(qws))
        ws = lbq._workspace(nws, "cuda")

        def fn():
            rc = lbq.lbq_linear_fwd_grouped(m, probs, len(qws), None if ws is None else ws.data_ptr(), nws,
                                            stream.cuda_stream)
            assert rc == 0, rc
    elif kind == "decode" or kind == "train":
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=1, outlier_frac=0.001, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W)
        del W
        if kind == "decode":
            m = int(arg[1:])
            X = syn.normal_bf16((m, k), 1.0, seed=2, device="cuda")
            fn = lambda: lbq.linear_fwd(X, qw)
        else:
            m, r, s = 4096, 16, 2.0
            X = syn.normal_bf16((m, k), 1.0, seed=2, device="cuda")
            A = syn.normal_bf16((r, k), 0.01, seed=3, device="cuda")
            B = syn.normal_bf16((n, r), 0.01, seed=4, device="cuda")
            dY = syn.normal_bf16((m, n), 0.1, seed=5, device="cuda")
            _, T = lbq.linear_fwd(X, qw, A, B, s)
            _, U = lbq.linear_bwd(dY, qw, A, B, s)
            fn = {"fwd": lambda: lbq.linear_fwd(X, qw, A, B, s),
                  "bwd": lambda: lbq.linear_bwd(dY, qw, A, B, s),
                  "grads": lambda: lbq.lora_grads(X, dY, T, U, s)}[arg]
    elif kind == "traingrp":
        # gate and up at M = 4096, rank 16, as one grouped call (arg: fwd or bwd)
        m, r, s = 4096, 16, 2.0
        fwd_p, bwd_p = [], []
        for i, nm in enumerate(("gate", "up")):
            n, k = syn.LLAMA3_8B_SHAPES[nm]
            W = syn.weight_bf16(n, k, 0.02, seed=1 + i, outlier_frac=0.001, device="cuda")
            qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W)
            del W
            X = syn.normal_bf16((m, k), 1.0, seed=2 + i, device="cuda")
            A = syn.normal_bf16((r, k), 0.01, seed=3 + i, device="cuda")
            B = syn.normal_bf16((n, r), 0.01, seed=4 + i, device="cuda")
            dY = syn.normal_bf16((m, n), 0.1, seed=5 + i, device="cuda")
            fwd_p.append((X, qw, A, B, s))
            bwd_p.append((dY, qw, A, B, s))
        fn = {"fwd": lambda: lbq.linear_fwd_grouped(fwd_p), "bwd": lambda: lbq.linear_bwd_grouped(bwd_p)}[arg]
    elif kind == "codebook70b":
        n, k = syn.LLAMA3_70B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.015, seed=1, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "codebook", double_quant=True, codebook=syn.codebook_normal16()).quantize(W)
        del W
        m = int(arg[1:])
        X = syn.normal_bf16((m, k), 1.0, seed=2, device="cuda")
        fn = lambda: lbq.linear_fwd(X, qw)
    elif kind == "merge":
        # merging a rank-16 adapter into one 8B matrix (INT4 g128 -> bf16)
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=1, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4).quantize(W)
        A = syn.normal_bf16((16, k), 0.01, seed=3, device="cuda")
        B = syn.normal_bf16((n, 16), 0.01, seed=4, device="cuda")
        fn = lambda: lbq.merge_lora(qw, A, B, 2.0, out=W)
    elif kind == "select":
        # choosing the INT4 quarter of one 8B matrix's channels (128 calibration tokens)
        n, k = syn.LLAMA3_8B_SHAPES[name]
        W = syn.weight_bf16(n, k, 0.02, seed=1, device="cuda")
        Xc = syn.normal_bf16((128, k), 1.0, seed=2, device="cuda")
        fn = lambda: lbq.channel_mix_select(W, Xc, n // 4)
    elif kind == "quantize":
        n, k = (syn.LLAMA3_8B_SHAPES.get(name) or syn.LLAMA3_70B_SHAPES[name])
        W = syn.weight_bf16(n, k, 0.02, seed=1, device="cuda")
        qw = lbq.QuantizedWeight(n, k, "minmax", 4) if arg == "int4" else \
            lbq.QuantizedWeight(n, k, "codebook", double_quant=True, codebook=syn.codebook_normal16())
        fn = lambda: qw.quantize(W)
    else:
        raise SystemExit(f"unknown case {args.case}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(args.reps - 1):
        fn()
    e0.record(stream)
    fn()
    e1.record(stream)
    torch.cuda.synchronize()
    print(json.dumps({"case": args.case, "ms_last_call": round(e0.elapsed_time(e1), 4),
                      "device_status": lbq.device_status()}))
    return 0


# ----------------------------------------------------------------------------- main
def main():
    args = parse_args()
    if args.case:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args)
    # CPU baseline first (before any CUDA work; OpenMP threads of the oracle)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    import torch
    from qlora_quantized_linear_b200 import lbq, synthetic as syn
    dist = Dist()
    peaks = measured_peaks()
    wl, value, ms, clocks, roofline, per_matrix, e2e = run_decode(args, dist, lbq, syn, torch, peaks)
    rows = {}
    if args.rows == "all":
        stream = torch.cuda.Stream()
        del wl
        torch.cuda.empty_cache()
        for key, fn in (("train_8b_mlp_M4096_r16", row_training), ("codebook_70b_dq", row_codebook70b),
                        ("mixed_8b", row_mixed), ("quantize_8b_int4", row_quantize8b),
                        ("merge_8b_r16", row_merge8b), ("channel_select_8b", row_channel_select)):
            try:
                rows[key] = fn(lbq, syn, torch, peaks, stream)
            except Exception as e:  # report, do not hide, a failing row
                rows[key] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
    status = lbq.device_status()
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "LLaMA-3-8B layer set (q,k,v,o 4096/1024x4096; gate,up 14336x4096; down 4096x14336), "
                               "INT4 g128 MinMax, forward dequant-GEMM at M=1 and M=16 per step",
                   "weights": "N(0, 0.02^2) bf16, 0.1% input channels x20, 7 seeded copies",
                   "l2": "7 rotating weight copies (116 MB per pass > one pass of L2 reuse; a copy returns every 7th pass)",
                   "launch": "one CUDA graph per step: 2 grouped decode GEMV launches (M=1 and M=16, 7 layers each) back to back (programmatic dependent launch); per_matrix from separate probe graphs with events between single-matrix calls",
                   "parallelism": f"replicas x{dist.world}"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": args.steps * wl_calls(),
        "clocks": clocks, "per_matrix": per_matrix, "rows": rows, "device_status": status,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def wl_calls():
    return len(DECODE_M)


if __name__ == "__main__":
    sys.exit(main())
