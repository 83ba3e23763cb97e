#!/usr/bin/env python
"""Benchmark of the W4A16 AWQ linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Metric: W4A16 GEMV HBM GB/s (% of peak) at M=1; GEMM TFLOP/s at M=2048.
  * value (first head): one step = one synthetic 8B-class decode token through the full stack of
    32 layers x 7 W4A16 linears (q, k, v, o, gate, up, down with Llama-3-8B shapes) at M=1, run back to
    back on one stream through w4a16_linear (GEMV mode), captured as one CUDA graph with programmatic
    dependent launch.  GB/s = algorithmic bytes per step (packed weights + scales + zeros + x' + y) over
    the device time of the step.  3.63 GB per step, far larger than the 126 MB L2, so every step streams
    from HBM.
  * gemm (second head): the three prefill shapes at M=2048 tokens through w4a16_gemm, TFLOP/s =
    2 M N K / device time (one step = the three shapes back to back, ~250 MB of operands > L2).
Inputs are synthetic (seeded torch CUDA generator; W ~ N(0, 0.02^2), activations N(0,1) with 1% of the
channels x20), quantized on the device with awq_act_scale / awq_pack / awq_apply_inv_scale.
With N > 1 GPUs every rank runs an independent replica (the layer needs no exchange); value is the
bytes of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV HBM GB/s (% of peak) at M=1; GEMM TFLOP/s at M=2048"
DECODE_SHAPES = [("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024), ("o", 4096, 4096),
                 ("gate", 4096, 14336), ("up", 4096, 14336), ("down", 14336, 4096)]  # (name, K, N)
# The same layer with the linears that share an input fused into one (the "fused modules" of the
# AutoAWQ page): q|k|v stacked along N (4096 -> 6144) and gate|up stacked along N (4096 -> 28672).
FUSED_SHAPES = [("qkv", 4096, 6144), ("o", 4096, 4096), ("gate_up", 4096, 28672), ("down", 14336, 4096)]
LAYERS = 32
PREFILL_SHAPES = [(4096, 14336), (14336, 4096), (4096, 4096)]  # (K, N)
PREFILL_M = 2048
CROSSOVER_SHAPES = [(8192, 28672), (28672, 8192)]  # (K, N), 70B-class MLP shapes
CROSSOVER_MS = [1, 2, 4, 8, 16, 32, 64, 128, 256]
BYTES_PER_WEIGHT = 0.5 + 2.0 / 128 + 0.5 / 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def gemv_bytes(M, N, K, g=128):
    """Algorithmic bytes of one W4A16 linear: packed weight + scales + zeros, x' and y."""
    return N * K * (0.5 + 2.5 / g) + 2 * M * K + 2 * M * N


def pack_bytes(N, K):
    """Algorithmic bytes of one pack: W and s read, packed weight, scales and zeros written."""
    return 2 * N * K + 2 * K + N * K * BYTES_PER_WEIGHT


def decode_step_bytes(M=1):
    return LAYERS * sum(gemv_bytes(M, N, K) for _, K, N in DECODE_SHAPES)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "gemv_kernel": ["weight_only_int4_05_b200/csrc/gemv.cu", "weight_only_int4_05_b200/csrc/common.cuh"],
    "gemm_kernel": ["weight_only_int4_05_b200/csrc/gemm.cu", "weight_only_int4_05_b200/csrc/common.cuh"],
    "pack_kernel": ["weight_only_int4_05_b200/csrc/pack.cu", "weight_only_int4_05_b200/csrc/common.cuh"],
}


def profiled_traffic(kernel, path=TRAFFIC_FILE):
    """DRAM bytes per launch of `kernel` recorded from an ncu capture (profiles/traffic.json), or None when
    the file lacks it or the kernel's sources changed since the counters were taken."""
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != source_hash(KERNEL_SOURCES[kernel]):
        return None
    return float(rec["bytes_per_launch"])


# ------------------------------------------------------------------------------- distributed plumbing
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float, group_backend_device=None) -> float:
    """Maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=group_backend_device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_value(bytes_per_rank_step: float, steps: int, world: int, max_seconds: float) -> float:
    """Whole-job GB/s: the bytes every rank processed over the slowest rank's time."""
    return bytes_per_rank_step * steps * world / max_seconds / 1e9


# ------------------------------------------------------------------------------- clocks sampling
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        return summarize_clock_lines(self.lines)


def summarize_clock_lines(lines):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, smax, reasons, power = [], [], set(), []
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for name, val in zip(names, parts[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------- GPU workloads
class DecodeStack:
    """32 layers x 7 packed linears, inputs x' and outputs y resident in HBM, one CUDA graph per step."""

    def __init__(self, device, seed=0, M=1, layers=LAYERS, inputs_fn=None, prefetch=False, fused=False,
                 inv_s_fused=False, silu=False, inv_s_two_pass=False):
        """inputs_fn(layer, linear, M, N, K) -> (W, xcal, x) fp16 device tensors; default: the seeded
        device generator of the synthetic workload.  prefetch: each call passes the next linear's packed
        weight as an L2 prefetch hint (w4a16_linear_pf).  fused: 4 linears per layer (FUSED_SHAPES).
        inv_s_fused: the resident activations are the raw x and every call is w4a16_gemv_s(x, s), which
        divides by the AWQ scale inside the kernel (no separate 1/s pass).  silu (with fused): the gate|up
        linear is packed by awq_pack_gate_up and called as w4a16_gate_up_silu, writing silu(gate) * up
        (14336 columns) instead of both projections.  inv_s_two_pass: the same raw activations, but every linear
        is the two launches awq_apply_inv_scale(x, s) then w4a16_linear (the unfused form of inv_s_fused)."""
        self.prefetch = prefetch
        self.two_pass = inv_s_two_pass
        inv_s_fused = inv_s_fused or inv_s_two_pass
        self.silu = silu and fused
        self.inv_s_fused = inv_s_fused
        layer_shapes = FUSED_SHAPES if fused else DECODE_SHAPES
        cfg = 6 if fused else 2  # tensor-id namespace of the synthetic inputs
        import torch
        import synth
        import weight_only_int4_05_b200 as W4

        self.W4, self.torch, self.device, self.M = W4, torch, device, M
        self.entries = []  # (packed weight, x' view, y view)
        self.s_list = []   # AWQ scales (inv_s_fused only)
        self.xp_list = []  # scaled activations formed every step (inv_s_two_pass only)
        shapes = [(li, name, K, N) for li in range(layers) for (name, K, N) in layer_shapes]
        self.h2d_elems = sum(M * K for _, _, K, _ in shapes)
        self.d2h_elems = sum(M * N for _, _, _, N in shapes)
        self.x_all = torch.empty(self.h2d_elems, dtype=torch.float16, device=device)
        self.y_all = torch.empty(self.d2h_elems, dtype=torch.float16, device=device)
        xo = yo = 0
        for idx, (li, name, K, N) in enumerate(shapes):
            j = layer_shapes.index((name, K, N))
            if inputs_fn is None:
                Wt, xcal, x = synth.device_linear_inputs(seed, synth.tensor_id(cfg, li, j, 0), M, N, K, device)
            else:
                Wt, xcal, x = inputs_fn(li, j, M, N, K)
            s = W4.awq_act_scale(xcal)
            gate_up = self.silu and name == "gate_up"
            if gate_up:  # rows [0, N/2) are the gate projection, [N/2, N) the up projection
                pw = W4.awq_pack_gate_up(Wt[:N // 2].contiguous(), Wt[N // 2:].contiguous(), s)
            else:
                pw = W4.awq_pack(Wt, s)
            xv = self.x_all[xo:xo + M * K].view(M, K)
            if inv_s_fused:
                xv.copy_(x)
                self.s_list.append(s)
            else:
                W4.awq_apply_inv_scale(x, s, out=xv)
            yv = self.y_all[yo:yo + M * N].view(M, N)
            if gate_up:
                yv = yv.reshape(-1)[:M * N // 2].view(M, N // 2)
            self.entries.append((pw, xv, yv, K, N))
            if self.two_pass:
                self.xp_list.append(torch.empty_like(xv))
            xo += M * K
            yo += M * N
            del Wt, xcal, x
        self.launches_per_step = sum(self._launches(K, N) for _, _, _, K, N in self.entries)
        if self.two_pass:
            self.launches_per_step += len(self.entries)  # one inv_scale_kernel per linear
        need = max(W4.w4a16_workspace_bytes(W4.MODE_LINEAR, M, N, K) for _, _, _, K, N in self.entries)
        W4.reserve_workspace(need, device)
        torch.cuda.synchronize(device)
        self.graph = None

    def _launches(self, K, N):
        W4 = self.W4
        if self.M <= W4.w4a16_gemv_max_m(N, K):  # GEMV passes: one for M <= 8, else passes of 16 rows
            return 1 if self.M <= 8 else (self.M + 15) // 16
        return 1

    def eager_step(self):
        n = len(self.entries)
        for i, (pw, xv, yv, _, _) in enumerate(self.entries):
            if self.two_pass:
                self.W4.awq_apply_inv_scale(xv, self.s_list[i], out=self.xp_list[i])
                self.W4.w4a16_linear(self.xp_list[i], pw, out=yv)
            elif self.inv_s_fused:
                self.W4.w4a16_gemv_s(xv, self.s_list[i], pw, out=yv)
            elif yv.shape[1] * 2 == pw.N and self.silu:
                self.W4.w4a16_gate_up_silu(xv, pw, out=yv)
            elif self.prefetch:  # the next linear of the step (the first one of the next step at the end)
                self.W4.w4a16_linear_pf(xv, pw, self.entries[(i + 1) % n][0], out=yv)
            else:
                self.W4.w4a16_linear(xv, pw, out=yv)

    def capture(self):
        torch = self.torch
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.eager_step()  # warm caches (occupancy queries, workspace) outside the capture
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.eager_step()
        torch.cuda.synchronize(self.device)

    def step(self):
        self.graph.replay()

    def bytes_per_step(self):
        extra = sum(2 * K for _, _, _, K, _ in self.entries) if self.inv_s_fused else 0  # the scale vectors
        # the gate|up SiLU call writes N / 2 outputs per row instead of N
        less = sum(self.M * N for pw, _, yv, _, N in self.entries if yv.shape[1] * 2 == N)
        return sum(gemv_bytes(self.M, N, K) for _, _, _, K, N in self.entries) + extra - less


class PrefillGemm:
    """The three M=2048 prefill shapes, one CUDA graph per step (all three back to back)."""

    def __init__(self, device, seed=0, M=PREFILL_M):
        import torch
        import synth
        import weight_only_int4_05_b200 as W4

        self.W4, self.torch, self.device, self.M = W4, torch, device, M
        self.entries = []
        for i, (K, N) in enumerate(PREFILL_SHAPES):
            Wt, xcal, x = synth.device_linear_inputs(seed, synth.tensor_id(3, 0, i, 0), M, N, K, device)
            s = W4.awq_act_scale(xcal)
            pw = W4.awq_pack(Wt, s)
            xp = W4.awq_apply_inv_scale(x, s)
            y = torch.empty((M, N), dtype=torch.float16, device=device)
            self.entries.append((pw, xp, y, K, N))
            del Wt, xcal, x
        need = max(W4.w4a16_workspace_bytes(W4.MODE_GEMM, M, N, K) for _, _, _, K, N in self.entries)
        W4.reserve_workspace(need, device)
        torch.cuda.synchronize(device)

    def eager_step(self):
        for pw, xp, y, _, _ in self.entries:
            self.W4.w4a16_gemm(xp, pw, out=y)

    def capture(self):
        torch = self.torch
        self.eager_step()
        torch.cuda.synchronize(self.device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.eager_step()
        torch.cuda.synchronize(self.device)

    def step(self):
        self.graph.replay()

    def flops_per_step(self):
        return sum(2.0 * self.M * N * K for _, _, _, K, N in self.entries)


def time_steps(step_fn, steps, warmup, device, sampler=None):
    """Device time of `steps` calls of step_fn (CUDA events on the current stream), max over ranks."""
    import torch

    for _ in range(warmup):
        step_fn()
    barrier(device)
    torch.cuda.synchronize(device)
    if sampler is not None:
        sampler.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(steps):
        step_fn()
    ev1.record()
    torch.cuda.synchronize(device)
    barrier(device)
    clocks = sampler.stop() if sampler is not None else None
    seconds = ev0.elapsed_time(ev1) / 1e3
    return reduce_max(seconds, device), clocks


def e2e_decode(stack, steps, warmup, device):
    """Same metric through the public API with host buffers: every step copies all 224 x' from pinned
    host memory, runs the graph, and reads all y back to pinned host memory."""
    import torch

    x_host = stack.x_all.cpu().pin_memory()
    y_host = torch.empty(stack.y_all.shape, dtype=torch.float16).pin_memory()

    def step():
        stack.x_all.copy_(x_host, non_blocking=True)
        stack.step()
        y_host.copy_(stack.y_all, non_blocking=True)

    seconds, _ = time_steps(step, steps, warmup, device)
    return seconds, x_host.numel() * 2, y_host.numel() * 2


# ------------------------------------------------------------------------------- CPU oracle legs
def oracle_sample_linears(seed=0):
    """Host inputs for the CPU legs: linears of the decode stack in layer order (host generator)."""
    import synth

    for li in range(LAYERS):
        for j, (name, K, N) in enumerate(DECODE_SHAPES):
            yield li, name, K, N, synth.linear_inputs(seed, 2, li, j, 1, N, K)


def oracle_time_linear(d, K, N):
    """Oracle seconds of one M=1 linear: (quantize + pack, matmul).  The matmul computes every output
    y[0][n] in fp64 from the quantized weight."""
    import numpy as np
    from oracle import oracle as O

    s = O.act_scale(d["xcal"].view(np.uint16))
    xp = O.inv_scale(d["x"].view(np.uint16), s)
    t0 = time.perf_counter()
    q, sc, z = O.quantize(d["W"].view(np.uint16), s)
    O.pack(q, sc, z)
    t1 = time.perf_counter()
    ms = np.zeros(N, np.int32)
    ns = np.arange(N, dtype=np.int32)
    O.linear_pairs_f64(xp, q, sc, z, ms, ns)
    return t1 - t0, time.perf_counter() - t1


def cpu_baseline(budget_s=12.0):
    """The oracle as it stands, single-threaded on this host, on the first linears of the decode stack
    until about `budget_s` seconds of matmul time; GB/s of the same algorithmic bytes.  Quantize + pack is
    timed separately (setup in the GPU arm as well) and reported beside it."""
    total_t = total_b = pack_t = pack_b = 0.0
    names = []
    for li, name, K, N, d in oracle_sample_linears():
        tp, tm = oracle_time_linear(d, K, N)
        pack_t += tp
        pack_b += pack_bytes(N, K)
        total_t += tm
        total_b += gemv_bytes(1, N, K)
        names.append(f"L{li}.{name}")
        if total_t >= budget_s:
            break
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "matmul_s": total_t,
            "pack": {"value": pack_b / pack_t / 1e9, "unit": "GB/s", "seconds": pack_t},
            "sample": f"{len(names)} linears of the M=1 decode stack ({names[0]}..{names[-1]}), "
                      f"{total_b / 1e6:.1f} MB of packed weight: fp64 matmul {total_t:.1f} s and quantize + pack "
                      f"{pack_t:.1f} s of single-thread oracle time, timed separately"}


REF_ROWS_PER_STEP = 256


def run_reference(args):
    """Reference arm: the CPU oracle on this host's cores.  One step = 256 outputs of the next M=1 linear
    of the decode stack (layer 0's q, k, v, o, gate, up, down, cycling) -- a bounded sample of the decode
    workload; GB/s counts the algorithmic bytes of exactly those outputs."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    from oracle import oracle as O

    prepared = []
    for li, name, K, N, d in oracle_sample_linears():
        s = O.act_scale(d["xcal"].view(np.uint16))
        xp = O.inv_scale(d["x"].view(np.uint16), s)
        q, sc, z = O.quantize(d["W"].view(np.uint16), s)
        prepared.append((K, N, xp, q, sc, z))
        if len(prepared) >= len(DECODE_SHAPES):
            break
    rows = REF_ROWS_PER_STEP

    def step(i):
        K, N, xp, q, sc, z = prepared[i % len(prepared)]
        ns = (np.arange(rows, dtype=np.int32) + (i * rows)) % N
        ms = np.zeros(rows, np.int32)
        t0 = time.perf_counter()
        O.linear_pairs_f64(xp, q, sc, z, ms, ns)
        return time.perf_counter() - t0, rows * K * BYTES_PER_WEIGHT + 2 * K + 2 * rows

    for i in range(args.warmup):
        step(i)
    tt = bb = 0.0
    for i in range(args.steps):
        t, b = step(i)
        tt += t
        bb += b
    value = bb / tt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "decode stack (32 layers x 7 Llama-3-8B-shaped W4A16 linears, M=1); each step "
                                   "a bounded sample: 256 outputs of the next linear of layer 0",
                       "M": 1, "rows_per_step": rows},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} steps x {rows} outputs, {bb / 1e6:.1f} MB of packed weight"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------------------- our arm
def gpu_uuid_id(device):
    import torch

    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        return str(device.index)


def time_graph_calls(calls, reps, warmup, device):
    """Device seconds per call of a list of launches captured as one CUDA graph and replayed `reps` times
    (each replay runs every call once), max over ranks."""
    import torch

    for c in calls:
        c()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    secs, _ = time_steps(g.replay, reps, warmup, device)
    del g
    return secs / reps / len(calls)


def weight_copies(W4, Wt, s, min_bytes):
    """Enough packed copies of one weight that together they exceed `min_bytes` (L2 defeated by rotation)."""
    N, K = Wt.shape
    per = N * K * BYTES_PER_WEIGHT
    n = max(2, int(-(-min_bytes // per)))
    return [W4.awq_pack(Wt, s) for _ in range(n)]


def measure_sweep(device, peaks, reps):
    """Config 1: each M=1 Llama-3-8B linear alone, calls over weight copies totalling 4 x L2, one graph."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    out = []
    for i, (name, K, N) in enumerate([("q/o", 4096, 4096), ("k/v", 4096, 1024), ("gate/up", 4096, 14336),
                                      ("down", 14336, 4096)]):
        Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(1, 0, i, 0), 1, N, K, device)
        s = W4.awq_act_scale(xcal)
        xp = W4.awq_apply_inv_scale(x, s)
        pws = weight_copies(W4, Wt, s, 512 * 2**20)
        del Wt, xcal, x
        y = torch.empty((1, N), dtype=torch.float16, device=device)
        ws = W4.reserve_workspace(max(256, W4.w4a16_workspace_bytes(W4.MODE_GEMV, 1, N, K)), device)
        calls = [(lambda p=pw: W4.w4a16_linear(xp, p, out=y, workspace=ws)) for pw in pws]
        sec = time_graph_calls(calls, reps, 3, device)
        gbs = gemv_bytes(1, N, K) / sec / 1e9
        out.append({"shape": name, "K": K, "N": N, "M": 1, "us": round(sec * 1e6, 3), "GB/s": round(gbs, 1),
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "copies": len(pws)})
        del pws
        torch.cuda.empty_cache()
    return out


def measure_tiny(device, reps):
    """Config 0: the tiny layer (M=1, K=512, N=256) -- latency-bound; microseconds per call in a graph."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(0, 0, 0, 0), 1, 256, 512, device)
    s = W4.awq_act_scale(xcal)
    xp = W4.awq_apply_inv_scale(x, s)
    pw = W4.awq_pack(Wt, s)
    y = torch.empty((1, 256), dtype=torch.float16, device=device)
    calls = [(lambda: W4.w4a16_linear(xp, pw, out=y))] * 64
    sec = time_graph_calls(calls, reps, 3, device)
    return {"shape": "tiny", "K": 512, "N": 256, "M": 1, "us": round(sec * 1e6, 3),
            "GB/s": round(gemv_bytes(1, 256, 512) / sec / 1e9, 2), "note": "latency-bound; weights stay in L2"}


def measure_pack(device, peaks, reps):
    """awq_pack on the gate/up weight (4096 -> 14336), two different weights alternating (235 MB of fp16
    input, more than L2); GB/s of W and s read plus the packed arrays written."""
    import synth
    import weight_only_int4_05_b200 as W4

    K, N = 4096, 14336
    inputs = []
    for i in range(2):
        Wt, xcal, _ = synth.device_linear_inputs(0, synth.tensor_id(1, 1, 2 + i, 0), 1, N, K, device)
        inputs.append((Wt, W4.awq_act_scale(xcal)))
    outs = [W4.awq_pack(*inputs[i]) for i in range(2)]
    calls = [(lambda i=i: W4.awq_pack(inputs[i][0], inputs[i][1], out=outs[i])) for i in range(2)]
    sec = time_graph_calls(calls, reps, 3, device)
    gbs = pack_bytes(N, K) / sec / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "us": round(sec * 1e6, 2), "K": K, "N": N,
            "frac": round(gbs / peaks["hbm_gbs"], 4), "kernel": "pack_kernel",
            "bytes_per_launch": pack_bytes(N, K), "traffic": profiled_traffic("pack_kernel"),
            "workload": "awq_pack of the 4096 -> 14336 weight, two weights alternating (inputs larger than L2)"}


def measure_groups(device, peaks, reps):
    """Group sizes 64 and 256: the M=1 decode shapes (calls over weight copies larger than L2, one graph) and
    the M=2048 prefill of the 4096 -> 14336 shape."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    out = []
    for g in (64, 256):
        for i, (name, K, N) in enumerate([("q/o", 4096, 4096), ("k/v", 4096, 1024), ("gate/up", 4096, 14336),
                                          ("down", 14336, 4096)]):
            Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(1, 0, i, 0), 1, N, K, device)
            s = W4.awq_act_scale(xcal)
            xp = W4.awq_apply_inv_scale(x, s)
            per = N * K * (0.5 + 2.5 / g)
            pws = [W4.awq_pack(Wt, s, g=g) for _ in range(max(2, int(-(-(512 * 2**20) // per))))]
            del Wt, xcal, x
            y = torch.empty((1, N), dtype=torch.float16, device=device)
            ws = W4.reserve_workspace(max(256, W4.w4a16_workspace_bytes(W4.MODE_GEMV, 1, N, K, g)), device)
            calls = [(lambda p=pw: W4.w4a16_linear(xp, p, out=y, workspace=ws)) for pw in pws]
            sec = time_graph_calls(calls, reps, 3, device)
            gbs = gemv_bytes(1, N, K, g) / sec / 1e9
            out.append({"g": g, "shape": name, "K": K, "N": N, "M": 1, "us": round(sec * 1e6, 3),
                        "GB/s": round(gbs, 1), "frac": round(gbs / peaks["hbm_gbs"], 4)})
            del pws
            torch.cuda.empty_cache()
        K, N, M = 4096, 14336, PREFILL_M
        Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(3, 0, 0, 0), M, N, K, device)
        s = W4.awq_act_scale(xcal)
        xp = W4.awq_apply_inv_scale(x, s)
        pw = W4.awq_pack(Wt, s, g=g)
        del Wt, xcal, x
        y = torch.empty((M, N), dtype=torch.float16, device=device)
        ws = W4.reserve_workspace(max(256, W4.w4a16_workspace_bytes(W4.MODE_GEMM, M, N, K, g)), device)
        sec = time_graph_calls([lambda: W4.w4a16_gemm(xp, pw, out=y, workspace=ws)], max(20, reps), 3, device)
        tf = 2.0 * M * N * K / sec / 1e12
        out.append({"g": g, "shape": "prefill gate/up", "K": K, "N": N, "M": M, "us": round(sec * 1e6, 2),
                    "TFLOP/s": round(tf, 1), "frac": round(tf / peaks["bf16_tflops"], 4)})
        del pw, xp, y
        torch.cuda.empty_cache()
    return out


def measure_int3(device, peaks, reps):
    """The packed 3-bit layout: the M=1 decode shapes through w3a16_gemv (calls over weight copies larger than
    L2, one graph); bytes counted at 0.375 + 2.5/128 per weight."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    out = []
    for i, (name, K, N) in enumerate([("q/o", 4096, 4096), ("k/v", 4096, 1024), ("gate/up", 4096, 14336),
                                      ("down", 14336, 4096)]):
        Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(1, 0, i, 0), 1, N, K, device)
        s = W4.awq_act_scale(xcal)
        xp = W4.awq_apply_inv_scale(x, s)
        per = N * K * (0.375 + 2.5 / 128)
        pws = [W4.awq_pack3(Wt, s) for _ in range(max(2, int(-(-(512 * 2**20) // per))))]
        del Wt, xcal, x
        y = torch.empty((1, N), dtype=torch.float16, device=device)
        ws = W4.reserve_workspace(max(256, W4.w4a16_workspace_bytes(W4.MODE_GEMV, 1, N, K)), device)
        calls = [(lambda p=pw: W4.w3a16_gemv(xp, p, out=y, workspace=ws)) for pw in pws]
        sec = time_graph_calls(calls, reps, 3, device)
        b = per + 2 * K + 2 * N
        out.append({"shape": name, "K": K, "N": N, "M": 1, "us": round(sec * 1e6, 3),
                    "GB/s": round(b / sec / 1e9, 1), "frac": round(b / sec / 1e9 / peaks["hbm_gbs"], 4),
                    "weights_per_s_G": round(N * K / sec / 1e9, 1)})
        del pws
        torch.cuda.empty_cache()
    return out


def measure_search(device, reps=3):
    """awq_search_scale on the 4096 -> 4096 projection with 512 calibration rows and 21 grid points, device
    time per search through the C entry point (preallocated buffers; no host synchronisation inside)."""
    import ctypes
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    N, K, R, n_grid = 4096, 4096, 512, 20
    Wt, xcal, _ = synth.device_linear_inputs(0, synth.tensor_id(8, 0, 0, 0), 1, N, K, device, rows=R)
    L = W4._lib.load()
    need = int(L.awq_search_workspace_bytes(N, K, R, 128, n_grid))
    ws = torch.empty(need, dtype=torch.uint8, device=device)
    losses = torch.empty(n_grid + 1, dtype=torch.float64, device=device)
    s = torch.empty(K, dtype=torch.float16, device=device)
    best = torch.empty(4, dtype=torch.int32, device=device)
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream(device).cuda_stream)

    def run():
        rc = L.awq_search_scale(P(Wt.data_ptr()), P(xcal.data_ptr()), N, K, R, 128, n_grid, P(losses.data_ptr()),
                                P(s.data_ptr()), P(best.data_ptr()), P(ws.data_ptr()), need, st)
        assert rc == 0, rc

    secs, _ = time_steps(run, reps, 1, device)
    per = secs / reps
    return {"value": round(per * 1e3, 3), "unit": "ms per search", "N": N, "K": K, "rows": R,
            "grid_points": n_grid + 1, "ms_per_grid_point": round(per * 1e3 / (n_grid + 1), 3),
            "best_alpha": int(best[0].item()) / n_grid,
            "workload": "AWQ scale search of one 4096 -> 4096 linear: per grid point the scale, awq_pack, 1/s, "
                        "the GEMM over 512 calibration rows and the fp64 squared error"}


def measure_gptq(device, reps=2):
    """gptq_quantize of the 4096 -> 4096 projection on 4096 calibration rows (device time per layer)."""
    import ctypes
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    N = K = R = 4096
    Wt, xcal, _ = synth.device_linear_inputs(0, synth.tensor_id(9, 0, 0, 0), 1, N, K, device, rows=R)
    L = W4._lib.load()
    need = int(L.gptq_workspace_bytes(N, K, R, 128))
    ws = torch.empty(need, dtype=torch.uint8, device=device)
    out = W4.awq_pack(Wt, None)
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream(device).cuda_stream)

    def run():
        rc = L.gptq_quantize(P(Wt.data_ptr()), P(xcal.data_ptr()), N, K, R, 128, ctypes.c_double(1e-6),
                             P(out.qweight.data_ptr()), P(out.scales.data_ptr()), P(out.qzeros.data_ptr()),
                             P(ws.data_ptr()), need, st)
        assert rc == 0, rc

    secs, _ = time_steps(run, reps, 1, device)
    per = secs / reps
    flops = R * K * K + 2 * K**3 / 3 + N * K * K  # Gram (lower half), Cholesky + inverse, lazy updates (fp64)
    return {"value": round(per * 1e3, 2), "unit": "ms per layer", "N": N, "K": K, "rows": R,
            "fp64_GFLOP": round(flops / 1e9, 1), "fp64_TFLOP/s": round(flops / per / 1e12, 2),
            "workload": "GPTQ of one 4096 -> 4096 linear on 4096 calibration rows into the W4A16 layout"}


def measure_crossover(device, reps):
    """Config 4: both modes at every M on the two 70B-class shapes; per M the faster mode and the one
    w4a16_linear picks (calls over weight copies larger than L2, one graph per point)."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    rows = []
    for i, (K, N) in enumerate(CROSSOVER_SHAPES):
        Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(4, 0, i, 0), max(CROSSOVER_MS), N, K, device)
        s = W4.awq_act_scale(xcal)
        xp_all = W4.awq_apply_inv_scale(x, s)
        pws = weight_copies(W4, Wt, s, 512 * 2**20)
        del Wt, xcal, x
        gmax = W4.w4a16_gemv_max_m(N, K)
        for M in CROSSOVER_MS:
            xp = xp_all[:M].contiguous()
            y = torch.empty((M, N), dtype=torch.float16, device=device)
            need = max(W4.w4a16_workspace_bytes(W4.MODE_GEMV, M, N, K), W4.w4a16_workspace_bytes(W4.MODE_GEMM, M, N, K))
            ws = W4.reserve_workspace(max(256, need), device)
            row = {"K": K, "N": N, "M": M}
            for mode, fn in (("gemv", W4.w4a16_gemv), ("gemm", W4.w4a16_gemm)):
                calls = [(lambda p=pw: fn(xp, p, out=y, workspace=ws)) for pw in pws]
                row[mode + "_us"] = round(time_graph_calls(calls, reps, 2, device) * 1e6, 2)
            row["faster"] = "gemv" if row["gemv_us"] <= row["gemm_us"] else "gemm"
            row["chosen"] = "gemv" if M <= gmax else "gemm"
            row["gemv_GB/s"] = round(gemv_bytes(M, N, K) / row["gemv_us"] / 1e3, 1)
            row["gemm_TFLOP/s"] = round(2.0 * M * N * K / row["gemm_us"] / 1e6, 1)
            rows.append(row)
        del pws
        torch.cuda.empty_cache()
    return rows


def run_gpu(args):
    import datetime
    import math

    import torch

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    import weight_only_int4_05_b200 as W4

    W4._lib.load()  # fails loudly if the CUDA library is missing
    peaks, peak_src = load_peaks()

    # ---- head 1: decode stack, GEMV mode
    stack = DecodeStack(device)
    stack.capture()
    sampler = ClockSampler(gpu_uuid_id(device))
    seconds, clocks = time_steps(stack.step, args.steps, args.warmup, device, sampler)
    bytes_step = stack.bytes_per_step()
    value = aggregate_value(bytes_step, args.steps, world, seconds)
    per_gpu = value / world
    launches = stack.launches_per_step
    roofline = {"bound": "hbm", "achieved": per_gpu, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": per_gpu / peaks["hbm_gbs"], "traffic": profiled_traffic("gemv_kernel"),
                "kernel": "gemv_kernel<1, XS, false, 128> (x' staged for gate/up, read directly for the others)",
                "peak_source": peak_src + " (HBM copy, burst)",
                "bytes_per_launch": bytes_step / launches, "launch_us": seconds / args.steps / launches * 1e6}

    # ---- e2e through the public API with host buffers
    e2e_steps = max(3, args.steps // 4)
    e2e_s, h2d, d2h = e2e_decode(stack, e2e_steps, max(3, args.warmup // 4), device)
    e2e_value = aggregate_value(bytes_step, e2e_steps, world, e2e_s)

    # ---- the same stack with the next linear's weights passed as an L2 prefetch hint
    stack.prefetch = True
    stack.capture()
    pf_s, pf_clocks = time_steps(stack.step, args.steps, args.warmup, device, ClockSampler(gpu_uuid_id(device)))
    pf_value = aggregate_value(bytes_step, args.steps, world, pf_s)
    decode_pf = {"value": pf_value, "unit": "GB/s", "ms_per_step": pf_s / args.steps * 1e3,
                 "frac": pf_value / world / peaks["hbm_gbs"], "steps": args.steps, "clocks": pf_clocks,
                 "workload": "the same decode stack; every call is w4a16_linear_pf with the next linear's packed "
                             "codes as the prefetch hint", "gpu_launches": launches * args.steps}

    # ---- the stack with q|k|v and gate|up fused (4 launches per layer, x' read once per fused linear)
    del stack
    torch.cuda.empty_cache()
    fstack = DecodeStack(device, fused=True)
    fstack.capture()
    f_s, f_clocks = time_steps(fstack.step, args.steps, args.warmup, device, ClockSampler(gpu_uuid_id(device)))
    f_bytes = fstack.bytes_per_step()
    f_value = aggregate_value(f_bytes, args.steps, world, f_s)
    decode_fused = {"value": f_value, "unit": "GB/s", "ms_per_step": f_s / args.steps * 1e3,
                    "frac": f_value / world / peaks["hbm_gbs"], "steps": args.steps, "clocks": f_clocks,
                    "bytes_per_step": f_bytes, "gpu_launches": fstack.launches_per_step * args.steps,
                    "workload": "decode stack with fused linears: 32 layers x {qkv 4096->6144, o 4096->4096, "
                                "gate_up 4096->28672, down 14336->4096}, M=1, w4a16_linear"}
    del fstack
    torch.cuda.empty_cache()

    # ---- the fused stack with the gate|up SiLU epilogue (the MLP's activation inside the gate|up call)
    ustack = DecodeStack(device, fused=True, silu=True)
    ustack.capture()
    u_s, u_clocks = time_steps(ustack.step, args.steps, args.warmup, device, ClockSampler(gpu_uuid_id(device)))
    u_bytes = ustack.bytes_per_step()
    u_value = aggregate_value(u_bytes, args.steps, world, u_s)
    decode_fused_silu = {"value": u_value, "unit": "GB/s", "ms_per_step": u_s / args.steps * 1e3,
                         "frac": u_value / world / peaks["hbm_gbs"], "steps": args.steps, "clocks": u_clocks,
                         "bytes_per_step": u_bytes, "gpu_launches": ustack.launches_per_step * args.steps,
                         "workload": "fused decode stack with w4a16_gate_up_silu: 32 layers x {qkv 4096->6144, "
                                     "o 4096->4096, gate|up+SiLU 4096->2x14336 writing 14336, down 14336->4096}"}
    del ustack
    torch.cuda.empty_cache()

    # ---- the plain stack with the AWQ 1/s fused into every GEMV (raw x and s in, no separate scaling pass)
    sstack = DecodeStack(device, inv_s_fused=True)
    sstack.capture()
    s_s, s_clocks = time_steps(sstack.step, args.steps, args.warmup, device, ClockSampler(gpu_uuid_id(device)))
    s_bytes = sstack.bytes_per_step()
    s_value = aggregate_value(s_bytes, args.steps, world, s_s)
    decode_inv_s = {"value": s_value, "unit": "GB/s", "ms_per_step": s_s / args.steps * 1e3,
                    "frac": s_value / world / peaks["hbm_gbs"], "steps": args.steps, "clocks": s_clocks,
                    "bytes_per_step": s_bytes, "gpu_launches": sstack.launches_per_step * args.steps,
                    "workload": "the plain decode stack with raw activations: every call is w4a16_gemv_s(x, s), "
                                "x / s formed inside the kernel (bit-identical x')"}
    del sstack
    torch.cuda.empty_cache()

    # ---- the same work unfused: awq_apply_inv_scale then w4a16_linear for every linear (448 launches per token)
    tstack = DecodeStack(device, inv_s_two_pass=True)
    tstack.capture()
    t_s, t_clocks = time_steps(tstack.step, args.steps, args.warmup, device, ClockSampler(gpu_uuid_id(device)))
    t_value = aggregate_value(s_bytes, args.steps, world, t_s)
    decode_inv_s_two_pass = {"value": t_value, "unit": "GB/s", "ms_per_step": t_s / args.steps * 1e3,
                             "frac": t_value / world / peaks["hbm_gbs"], "steps": args.steps, "clocks": t_clocks,
                             "bytes_per_step": s_bytes, "gpu_launches": tstack.launches_per_step * args.steps,
                             "workload": "the same raw activations, unfused: awq_apply_inv_scale then w4a16_linear "
                                         "for every linear (the same algorithmic bytes as decode_inv_s_fused)"}
    del tstack
    torch.cuda.empty_cache()

    # ---- head 2: prefill GEMM at M=2048, timed over at least 150 ms
    pre = PrefillGemm(device)
    pre.capture()
    probe_s, _ = time_steps(pre.step, 3, 3, device)
    g_steps = max(20, math.ceil(0.15 / (probe_s / 3)))
    g_sampler = ClockSampler(gpu_uuid_id(device))
    g_seconds, g_clocks = time_steps(pre.step, g_steps, 3, device, g_sampler)
    tflops = pre.flops_per_step() * g_steps * world / g_seconds / 1e12
    g_per_gpu = tflops / world
    per_shape = []
    for (pw, xp, y, K, N) in pre.entries:
        sec = time_graph_calls([(lambda pw=pw, xp=xp, y=y: W4.w4a16_gemm(xp, pw, out=y))], max(20, g_steps // 2), 3,
                               device)
        per_shape.append({"K": K, "N": N, "M": PREFILL_M, "us": round(sec * 1e6, 2),
                          "TFLOP/s": round(2.0 * PREFILL_M * N * K / sec / 1e12, 1)})
    gemm = {"value": tflops, "unit": "TFLOP/s", "ms_per_step": g_seconds / g_steps * 1e3, "steps": g_steps,
            "timed_ms": g_seconds * 1e3,
            "workload": "prefill GEMM M=2048: (K,N) = (4096,14336), (14336,4096), (4096,4096), one step = all three",
            "per_shape": per_shape, "gpu_launches": 3 * g_steps, "clocks": g_clocks,
            "roofline": {"bound": "tensor", "achieved": g_per_gpu, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": g_per_gpu / peaks["bf16_tflops"],
                         "frac_of_sustained": g_per_gpu / peaks["bf16_tflops_sustained"],
                         "traffic": profiled_traffic("gemm_kernel"), "kernel": "gemm_kernel",
                         "peak_source": peak_src + " (dense bf16 burst; fp16 runs at the bf16 tensor rate)"}}
    del pre
    torch.cuda.empty_cache()

    # ---- the other configurations: the M=1 sweep (config 1), the tiny layer (config 0), pack, crossover
    reps = max(5, min(50, args.steps // 4))
    sweep = measure_sweep(device, peaks, reps)
    tiny = measure_tiny(device, reps)
    pack = measure_pack(device, peaks, reps)
    crossover = None if args.no_crossover else measure_crossover(device, max(3, reps // 4))
    groups = measure_groups(device, peaks, reps)
    int3 = measure_int3(device, peaks, reps)
    search = measure_search(device)
    gptq = measure_gptq(device)

    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": seconds / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "pct_of_peak": 100.0 * per_gpu / peaks["hbm_gbs"],
            "config": {"workload": "decode stack: 32 layers x 7 W4A16 linears (Llama-3-8B shapes: q/o 4096->4096, "
                                   "k/v 4096->1024, gate/up 4096->14336, down 14336->4096), M=1, one token per step",
                       "M": 1, "layers": LAYERS, "group_size": 128, "bytes_per_step": bytes_step,
                       "l2": "inputs larger than L2 (3.63 GB of packed weights per step)",
                       "accumulate": "f32 (exact fp16 products on mma.sync, fp32 sums; scale applied in fp32)",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": roofline, "gpu_launches": launches * args.steps, "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gemm": gemm, "decode_sweep": sweep, "tiny": tiny, "pack": pack, "crossover": crossover,
            "decode_prefetch_hint": decode_pf, "decode_fused": decode_fused, "decode_inv_s_fused": decode_inv_s,
            "decode_inv_s_two_pass": decode_inv_s_two_pass,
            "decode_fused_silu": decode_fused_silu, "group_sizes": groups, "int3_layout": int3, "awq_search": search,
            "gptq": gptq}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    elif rank == 0:
        line["cpu_baseline"] = None
    status = W4.awq_last_device_status()
    if status != 0:
        line["device_status"] = status
    if world > 1:
        import torch.distributed as dist

        barrier(device)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


def run_profile_case(args):
    """One linear layer launched `warmup + steps` times eagerly on enough weight copies to exceed L2:
    the small case for detailed ncu captures.  spec = "gemv:K:N:M", "gemm:K:N:M", "silu:K:N:M" (gate|up
    with the SiLU epilogue, N = 2 NI) or "gptq:K:N:R" (one GPTQ per launch)."""
    import torch
    import synth
    import weight_only_int4_05_b200 as W4

    mode, K, N, M = args.profile_case.split(":")
    K, N, M = int(K), int(N), int(M)
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    W4._lib.load()
    launches = args.warmup + args.steps
    if mode == "gptq":  # one GPTQ of an N x K weight on M calibration rows per launch
        Wt, xcal, _ = synth.device_linear_inputs(0, synth.tensor_id(9, 0, 0, 0), 1, N, K, device, rows=M)
        for _ in range(launches):
            W4.gptq_quantize(Wt, xcal)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": args.profile_case, "launches": launches,
                          "device_status": W4.awq_last_device_status()}))
        return 0
    Wt, xcal, x = synth.device_linear_inputs(0, synth.tensor_id(5, 0, 0, 0), M, N, K, device)
    s = W4.awq_act_scale(xcal)
    xp = W4.awq_apply_inv_scale(x, s)
    copies = max(2, -(-256 * 2**20 // (N * K // 2)))  # > 2 x L2 of packed weights
    if mode == "silu":  # N = NI: the gate and up halves of a 2 NI x K weight
        pws = [W4.awq_pack_gate_up(Wt[:N // 2].contiguous(), Wt[N // 2:].contiguous(), s) for _ in range(copies)]
        y = torch.empty((M, N // 2), dtype=torch.float16, device=device)
    else:
        pws = [W4.awq_pack(Wt, s) for _ in range(copies)]
        y = torch.empty((M, N), dtype=torch.float16, device=device)
    del Wt, xcal, x
    fn = {"gemv": W4.w4a16_gemv, "gemm": W4.w4a16_gemm, "silu": W4.w4a16_gate_up_silu}[mode]
    for i in range(launches):
        fn(xp, pws[i % copies], out=y)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile_case, "launches": launches,
                      "copies": copies, "device_status": W4.awq_last_device_status()}))
    return 0


def run_crossover(args):
    """Both modes at every M of the crossover sweep (measure_crossover); prints one JSON line, no bench metric."""
    import torch
    import weight_only_int4_05_b200 as W4

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    W4._lib.load()
    rows = measure_crossover(device, max(3, args.steps))
    print(json.dumps({"crossover": rows, "gemv_max_m": W4.w4a16_gemv_max_m(8192, 28672),
                      "device_status": W4.awq_last_device_status()}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-crossover", action="store_true", help="leave the crossover sweep out of the bench line")
    ap.add_argument("--crossover", action="store_true",
                    help="time both modes at M = 1..256 on the 70B-class shapes (validates the mode choice)")
    ap.add_argument("--profile-case", default=None, metavar="MODE:K:N:M",
                    help="launch one linear (gemv or gemm) warmup+steps times for an ncu capture, no timing")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch N > 1 ranks with "
                         f"python -m torch.distributed.run --nproc-per-node N bench.py --gpus N\n")
        return 2
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return run_profile_case(args)
    if args.crossover:
        return run_crossover(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
