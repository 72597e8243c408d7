#!/usr/bin/env python
"""Benchmark of the codebook-VQ linear layer on B200 (one JSON line on stdout).

Metric: vq_linear microseconds per layer (one layer = one weight matrix, i.e. one
vq_linear_forward) and the achieved HBM bandwidth against the roofline at batch 1
and 16; TFLOP/s on the tensor-core path at M = 256.

Headline workload (``--workload llama3-8b-mlp``, the default): the Llama-3-8B MLP
shapes (gate and up 14336 x 4096, down 4096 x 14336), 2-stage RVQ 12+4 bits with
block-64 fp16 scales, bf16 activations, batch 1.  One step = gate, up and down
forward on one batch of input.  Other workloads are measured in the same run
and reported under "detail" (the SmolLM-135M-shaped 30-layer stack at M=1 and
16, the rotated 16-bit-index layer, batch 16 of the MLP, and M=256 of the
8192 x 8192 prefill tile on the tensor-core path).

Timing: W untimed warm-up steps; then exactly K steps bracketed by one pair of
CUDA events on the launching stream.  The steps are replays of CUDA graphs: one
graph holds a step on each weight copy in turn (whole cycles), single-step
graphs make up the rest, so K is exact.
The inputs are larger than L2: the step's weights exist in R device copies
(R x the step's weight bytes >= 4 x the L2 size) and step k runs on copy k mod R,
so every timed step reads weights that are not in L2, as the layers of a deep
model do, while the kernels' own code stays cached.  Barrier + synchronize
before and after; the max over ranks is reported.  With --gpus N (torchrun) every rank runs an independent replica
(the layer does not shard here) and ``value`` aggregates all ranks' layers.

``--impl reference`` times the CPU oracle (oracle/, plain C in fp64) on a bounded
row sample of the same workload and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import (CONFIGS, DT_BF16, DT_F16, FMT_VQ16, FMT_VQ16_RVQ, LayerSpec, make_correction,  # noqa: E402
                   make_layer, make_signs, make_x)

METRIC = "vq_linear µs/layer & achieved HBM GB/s (% of roofline) at batch 1/16; TFLOP/s at M=256"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "llama3-8b-mlp": dict(cfg=4, layers=1, gate_up_concurrent=True),
    "smollm-135m-stack": dict(cfg=2, layers=30),
    "vq16-4096-rht": dict(cfg=3, layers=1),
    "prefill-8192": dict(cfg=5, layers=1),
    "single-256": dict(cfg=1, layers=1),
}
# The residual bit-width ladder (GLQ README, "Bit widths": 3 bpw = 16 + 8, 4 = 16 + 16,
# 5 = 16 + 16 + 8) on a 4096 x 4096 layer with one scale per row, like the 16-bit
# workload; seeded with its own id.
for _bpw in (3, 4, 5):
    WORKLOADS[f"vq16-ladder-4096-{_bpw}bpw"] = dict(
        cfg=100 + _bpw, layers=1,
        config=dict(name=f"vq16-ladder-4096x4096-{_bpw}bpw", layers=1, act=DT_F16, Ms=(1, 8), rht=False,
                    tensors=[("w", LayerSpec(4096, 4096, FMT_VQ16_RVQ, 4096, bpw=_bpw))]))
# The MLP with a sparse correction sidecar on every matrix (orka README, "How it works":
# "(+ sparse correction)"): 0.1 % of the weights corrected, fp16 values ~ N(0, 0.05^2).
WORKLOADS["llama3-8b-mlp-corr"] = dict(cfg=4, layers=1, gate_up_concurrent=True, corr_density=0.001)
_16BIT = (FMT_VQ16, FMT_VQ16_RVQ)


def _workload_config(name):
    w = WORKLOADS[name]
    return w["config"] if "config" in w else CONFIGS[w["cfg"]]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def corr_bytes(L):
    """Bytes of a layer's sparse correction sidecar: row pointers, and a column (int32) and
    a value (fp16) per entry; 0 without one."""
    if L is None or not getattr(L, "corr", 0):
        return 0
    t = L.t
    return t["corr_rows"].numel() * 4 + (t["corr_cols"].numel() * 6 if "corr_cols" in t else 0)


def layer_bytes(spec, M, act_bytes=2):
    """Algorithmic bytes of one forward: planes + scales + codebooks + x + y (each once)."""
    G = spec.K // 8
    if spec.fmt == FMT_VQ16:
        planes, cb = spec.N * G * 2, 65536 * 16
    elif spec.fmt == FMT_VQ16_RVQ:  # one 16-bit plane and codebook per 16-bit stage, the 8-bit ones
        n16, n8 = spec.bpw // 2, spec.bpw % 2
        planes, cb = spec.N * G * (2 * n16 + n8), 65536 * 16 * n16 + 256 * 16 * n8
    else:
        planes = spec.N * G + spec.N * G // 2 + (spec.N * G // 2 if spec.fmt == 2 else 0)
        cb = 4096 * 16 + (256 if spec.fmt == 2 else 0)
    scales = spec.N * (spec.K // spec.scale_group) * 2
    return planes + scales + cb + M * spec.K * act_bytes + M * spec.N * act_bytes


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20",
                 "-i", str(self.gpu)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], parts[4]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- GPU arm

class Workload:
    """A workload's layers resident on the GPU plus chained activation buffers."""

    def __init__(self, name, max_M, seed=0, replicas=None):
        import torch

        import compressed_index_matmul_b200 as vq

        self.name = name
        w = WORKLOADS[name]
        self.cfg = w["config"] if "config" in w else CONFIGS[w["cfg"]]
        self.act = self.cfg["act"]
        self.tdtype = torch.bfloat16 if self.act == DT_BF16 else torch.float16
        self.max_M = max_M
        self.layers = []  # (label, spec, VQLinear)
        for li in range(w["layers"]):
            for ti, (label, spec) in enumerate(self.cfg["tensors"]):
                arr = make_layer(spec, cfg_id=w["cfg"], layer=li, tensor_id=ti, seed=seed)
                if w.get("corr_density"):
                    arr["corr"] = make_correction(spec.N, spec.K, density=w["corr_density"], cfg_id=w["cfg"],
                                                  layer=li, tensor_id=ti, seed=seed)
                L = vq.VQLinear(spec.N, spec.K, spec.fmt, spec.scale_group, self.act, max_M, arr,
                                rht=int(self.cfg["rht"]))
                self.layers.append((f"{li}.{label}", spec, L))
        # Copies of every layer's device arrays, cycled step by step so that the
        # weights a step reads are never in L2 (their total is >= 4x the L2 size);
        # the copies share the handle (forwards run one after another).
        if replicas is None:
            l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
            replicas = max(1, -(-4 * l2 // max(1, self.weight_bytes())))
        self.replicas = [self.layers]
        for _ in range(1, replicas):
            self.replicas.append([(name, spec, _clone_layer(L)) for name, spec, L in self.layers])
        # An MLP's gate and up projections read the same x and are independent: a step
        # issues them concurrently on two streams, each limited to half of the SMs
        # (vq_linear_set_sm_budget), then the down projection.
        self.role = {id(L): name.split(".")[1] for rep in self.replicas for name, _, L in rep}
        self.concurrent_gate_up = any(self.role[id(L)] == "gate" for _, _, L in self.layers) and \
            w.get("gate_up_concurrent", False)
        self.side = torch.cuda.Stream()
        self.sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        self.rht = self.cfg["rht"]
        K0 = self.layers[0][1].K
        self.x0 = torch.from_numpy(make_x(max_M, K0, self.act, cfg_id=w["cfg"], seed=seed).view(np.int16)).cuda() \
            .view(self.tdtype)
        if self.rht:
            self.signs = torch.from_numpy(make_signs(K0, cfg_id=w["cfg"], seed=seed)).cuda()
        self.outs = {}

    def weight_bytes(self):
        """Bytes of one copy of the step's layer inputs that do not depend on M."""
        return sum(layer_bytes(spec, 0) + corr_bytes(L) for _, spec, L in self.layers)

    def plan(self, M, replica=0):
        """Forward calls of one step: (layer, input tensor, output tensor) with the stack's chaining."""
        import torch

        calls = []
        x = self.x0[:M]
        prev_by_width = {}
        for name, spec, L in self.replicas[replica]:
            label = name.split(".")[1]
            key = (name, M)
            if key not in self.outs:
                self.outs[key] = torch.empty((M, spec.N), dtype=self.tdtype, device="cuda")
            y = self.outs[key]
            if label in ("q", "k", "v", "gate", "up", "w"):
                inp = x if spec.K == x.shape[1] else prev_by_width[spec.K]
            else:  # o / down read the most recent output of their input width
                inp = prev_by_width.get(spec.K, x)
            calls.append((L, inp, y))
            prev_by_width[spec.N] = y
            if label in ("o",):
                x = y  # next sub-block reads o's output
            if label == "down":
                x = y
        return calls

    def _forward(self, L, inp, y, stream):
        """One forward on `stream` (a raw cudaStream_t: the caller looks the stream up once
        per step instead of once per call)."""
        if self.rht:  # the layer rotates its input (vq_linear_forward_rotated)
            L.forward_rotated(inp, self.signs, y, stream)
        else:
            L.forward(inp, y, stream)

    def _pair(self, a, b):
        return (self.concurrent_gate_up and self.role[id(a[0])] == "gate" and self.role[id(b[0])] == "up"
                and a[1] is b[1])

    def enqueue(self, calls, M, events=None, concurrent=True):
        """Enqueue one step on the current stream.  With `events` (per-forward timing) or
        `concurrent` false every forward runs alone on the current stream; otherwise gate
        and up run concurrently."""
        import torch

        cur = torch.cuda.current_stream()
        cur_s = cur.cuda_stream
        i = 0
        while i < len(calls):
            if concurrent and events is None and i + 1 < len(calls) and self._pair(calls[i], calls[i + 1]):
                (g, gi, gy), (u, ui, uy) = calls[i], calls[i + 1]
                half = self.sms // 2
                g.set_sm_budget(half)
                u.set_sm_budget(self.sms - half)
                self.side.wait_stream(cur)
                self._forward(u, ui, uy, self.side.cuda_stream)
                self._forward(g, gi, gy, cur_s)
                cur.wait_stream(self.side)
                g.set_sm_budget(0)
                u.set_sm_budget(0)
                i += 2
                continue
            if events is not None:
                events[i].record()
            self._forward(*calls[i], cur_s)
            i += 1
        if events is not None:
            events[len(calls)].record()

    def rotation_fused(self, spec, M):
        """True where vq_linear_forward_rotated is one kernel: the automatic choice is the
        16-bit gather kernel (M <= 4), which rotates x itself."""
        mt = 1 if M <= 1 else 2 if M <= 2 else 4
        return (M <= 4 and spec.fmt in _16BIT and spec.K % 128 == 0 and spec.K <= 16384 and mt * spec.K <= 32768
                and spec.N % 4 == 0)

    def launches_per_step(self, M):
        n = 0
        for _, spec, L in self.layers:
            n += L.launches(M) + (1 if self.rht and not self.rotation_fused(spec, M) else 0)
        return n

    def bytes_per_step(self, M):
        # an unfused rotation reads and writes x once more (2 + 2 bytes per element)
        extra = sum(4 * M * spec.K for _, spec, _ in self.layers if self.rht and not self.rotation_fused(spec, M))
        return sum(layer_bytes(spec, M) + corr_bytes(L) for _, spec, L in self.layers) + extra

    def flops_per_step(self, M):
        return sum(2.0 * M * spec.N * spec.K for _, spec, _ in self.layers)


def _clone_layer(L):
    """A VQLinear sharing L's handle but reading its own copy of the device arrays."""
    import copy

    from compressed_index_matmul_b200 import _binding as B

    c = copy.copy(L)
    # The 65,536-entry codebooks of the 16-bit formats are tables shared by every
    # copy: GLQ's lattice codebook is shared by all layers and served from L2 (the
    # ladder's residual and 8-bit codebooks likewise).  The index planes, scales and
    # 4096-entry codebooks are copied.
    shared = ("cb1", "cbr", "cb8") if L.fmt in _16BIT else ()
    c.t = {k: (v if k in shared else v.clone()) for k, v in L.t.items()}
    c.planes = B.make_planes(c.t.get("lo"), c.t.get("hi4"), c.t.get("s2"), c.t.get("idx16"), c.t.get("idx8"),
                             c.t.get("corr_rows"), c.t.get("corr_cols"), c.t.get("corr_vals"))
    c.codebooks = L.codebooks if L.fmt in _16BIT else B.make_codebooks(c.t["cb1"], c.t.get("cb2"))
    c.close = lambda: None  # the handle belongs to L
    return c


L2_NOTE = "inputs larger than L2: the step's weights are cycled over {r} copies ({mb:.0f} MB, >= 4x L2)"


def capture_steps(wl, M, stream, evs=None, concurrent=True):
    """One CUDA graph per weight copy, each holding one step's forwards."""
    import torch

    graphs = []
    for r in range(len(wl.replicas)):
        calls = wl.plan(M, r)
        with torch.cuda.stream(stream):
            wl.enqueue(calls, M, concurrent=concurrent)  # plain run: every call validated outside capture
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            wl.enqueue(calls, M, evs, concurrent=concurrent)
        graphs.append(g)
    return graphs


def capture_cycle(wl, M, stream, concurrent=True):
    """One CUDA graph holding one step on each weight copy in turn (R steps back to back)."""
    import torch

    g = torch.cuda.CUDAGraph()
    plans = [wl.plan(M, r) for r in range(len(wl.replicas))]
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        for calls in plans:
            wl.enqueue(calls, M, concurrent=concurrent)
    return g


def run_steps(graphs, cycle, first, steps, stream):
    """Enqueue exactly `steps` steps starting at step index `first`: whole cycles by the
    cycle graph where they line up, single-step graphs for the rest."""
    R = len(graphs)
    k = first
    end = first + steps
    while k < end:
        if k % R == 0 and end - k >= R:
            cycle.replay()
            k += R
        else:
            graphs[k % R].replay()
            k += 1


WARMUP_SECONDS = 0.5  # replays before any timed region, whatever --warmup is
REGIONS = 5           # timed regions of exactly K steps each; the line reports their median


def warm_up(graphs, cycle, stream, steps, seconds=WARMUP_SECONDS):
    """`steps` untimed steps, then more whole cycles until `seconds` of wall time have passed
    (clocks, L2 and TLB state settle before the first timed region).  Returns the next step index."""
    import torch

    with torch.cuda.stream(stream):
        run_steps(graphs, cycle, 0, steps, stream)
    stream.synchronize()
    k = steps
    R = len(graphs)
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        with torch.cuda.stream(stream):
            start = -(-k // R) * R  # next cycle boundary
            run_steps(graphs, cycle, k, start - k + R, stream)
            k = start + R
        stream.synchronize()
    return k


def timed_regions(graphs, cycle, stream, first, steps, regions):
    """`regions` back-to-back event regions of exactly `steps` steps each; ms per region."""
    import torch

    evs = [torch.cuda.Event(enable_timing=True) for _ in range(regions + 1)]
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        k = first
        for i in range(regions):
            run_steps(graphs, cycle, k, steps, stream)
            k += steps
            evs[i + 1].record(stream)
    stream.synchronize()
    return [evs[i].elapsed_time(evs[i + 1]) for i in range(regions)]


def time_graph(wl, M, steps, warmup, per_kernel=False, concurrent=True):
    """Replay the step graphs `steps` times (cycling the weight copies); per-step ms (and per-forward ms)."""
    import torch

    stream = torch.cuda.Stream()
    n = len(wl.plan(M))
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)] if per_kernel else None
    graphs = capture_steps(wl, M, stream, evs, concurrent=concurrent)
    R = len(graphs)
    per_fwd = np.zeros(n) if per_kernel else None
    if per_kernel:  # one step at a time, events between the forwards
        with torch.cuda.stream(stream):
            for k in range(warmup):
                graphs[k % R].replay()
            stream.synchronize()
            for k in range(steps):
                graphs[(warmup + k) % R].replay()
                stream.synchronize()
                per_fwd += np.array([evs[i].elapsed_time(evs[i + 1]) for i in range(n)])
        del graphs
        return None, per_fwd / steps
    cycle = capture_cycle(wl, M, stream, concurrent=concurrent)
    k = warm_up(graphs, cycle, stream, warmup, seconds=0.2)
    region_ms = timed_regions(graphs, cycle, stream, k, steps, 3)
    del graphs, cycle
    return [statistics.median(region_ms) / steps] * steps, None


def time_e2e(wl, M, steps, warmup):
    """Public API end to end: pinned-host x -> device, eager vq_linear_forward calls one after
    another on one stream, y -> pinned host."""
    import torch

    stream = torch.cuda.Stream()
    plans = [wl.plan(M, r) for r in range(len(wl.replicas))]
    calls = plans[0]
    src = wl.x0[:M]
    host_x = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
    host_x.copy_(src.cpu())
    last = calls[-1][2]
    host_y = torch.empty(last.shape, dtype=last.dtype, pin_memory=True)
    dev_x = wl.x0
    ms = []
    with torch.cuda.stream(stream):
        for k in range(warmup + steps):
            calls = plans[k % len(plans)]
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dev_x[:M].copy_(host_x, non_blocking=True)
            wl.enqueue(calls, M, concurrent=False)  # eager calls on one stream (no fork / join per step)
            host_y.copy_(last, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if k >= warmup:
                ms.append(e0.elapsed_time(e1))
    return ms, host_x.numel() * host_x.element_size(), host_y.numel() * host_y.element_size()


def measure(wl, M, steps, warmup, peaks, with_kernels=True, gpu_index=None):
    if gpu_index is not None:  # clocks and throttle reasons while this row is timed
        with ClockSampler(gpu_index) as clk:
            ms, per_fwd = time_graph(wl, M, steps, warmup, per_kernel=False)
        clocks = clk.summary()
    else:
        ms, per_fwd = time_graph(wl, M, steps, warmup, per_kernel=False)
        clocks = None
    res = {"M": M, "ms_per_step": statistics.fmean(ms), "layers_per_step": len(wl.layers)}
    res["us_per_layer"] = 1e3 * res["ms_per_step"] / len(wl.layers)
    b = wl.bytes_per_step(M)
    res["bytes_per_step"] = b
    res["hbm_gbs"] = b / (res["ms_per_step"] * 1e-3) / 1e9
    res["hbm_frac"] = res["hbm_gbs"] / peaks["hbm_gbs"]
    res["tflops"] = wl.flops_per_step(M) / (res["ms_per_step"] * 1e-3) / 1e12
    if clocks is not None:
        res["clocks"] = clocks
    if with_kernels:
        _, per_fwd = time_graph(wl, M, max(5, min(steps, 50)), 2, per_kernel=True)
        res["per_forward_us"] = [float(1e3 * v) for v in per_fwd]
    return res


def gpu_arm(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import compressed_index_matmul_b200 as vq
    from compressed_index_matmul_b200 import build as libbuild

    if rank == 0 or world == 1:
        libbuild.build()
    if world > 1:
        dist.barrier()
    vq.load()
    peaks, peak_src = load_peaks()
    M = args.batch
    wl = Workload(args.workload, max_M=max(M, 16))
    R = len(wl.replicas)

    # ------------------------------------------------ timed regions (exactly K steps each)
    stream = torch.cuda.Stream()
    graphs = capture_steps(wl, M, stream)
    cycle = capture_cycle(wl, M, stream)
    first = warm_up(graphs, cycle, stream, args.warmup)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v for v in vis.split(",") if v.strip()]
    smi_index = int(ids[local]) if local < len(ids) and ids[local].strip().isdigit() else local
    with ClockSampler(smi_index) as clk:
        region_ms = timed_regions(graphs, cycle, stream, first, args.steps, args.regions)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    del graphs, cycle
    layers = len(wl.layers)
    ms_per_step, us_per_layer = aggregate_over_ranks(float(statistics.median(region_ms)), args.steps, layers, world)

    # ------------------------------------------------ per-launch roofline (same stream)
    _, per_fwd = time_graph(wl, M, min(args.steps, 200), 3, per_kernel=True)  # event nodes between forwards
    launches_per_fwd = [L.launches(M) for _, _, L in wl.layers]
    bytes_per_fwd = [layer_bytes(spec, M) + corr_bytes(L) for _, spec, L in wl.layers]
    # When every forward runs the same single kernel (no rotation launch), a region's
    # time per launch is that kernel's average duration; else use the event nodes
    # captured between the forwards (which include the gaps).  A step that overlaps
    # gate and up has no such per-launch time, so the same forwards are timed one after
    # another (each with every SM) in a region of their own for the roofline.
    fused = all(wl.rotation_fused(spec, M) for _, spec, _ in wl.layers)
    uniform = (not wl.rht or fused) and len(set(launches_per_fwd)) == 1
    if uniform and wl.concurrent_gate_up:
        fwd_ms = time_graph(wl, M, args.steps, args.warmup, concurrent=False)[0][0] / len(wl.layers)
        launch_source = ("a separate region of K steps with the forwards one after another on one stream, every "
                         "SM each (every launch is this kernel) / launches")
    elif uniform:
        fwd_ms = ms_per_step / len(wl.layers)
        launch_source = ("timed region / launches (every launch is this kernel)" if launches_per_fwd[0] == 1 else
                         "timed region / forwards")
    else:
        fwd_ms = float(np.mean(per_fwd))
        launch_source = "CUDA event nodes between the forwards"
    per_fwd_eff = [fwd_ms / max(1, launches_per_fwd[0]) if uniform else fwd_ms] * len(wl.layers)
    achieved = sum(bytes_per_fwd) / (sum(per_fwd_eff) * 1e-3) / 1e9
    # the kernel the library plans for the first weight matrix (the step's largest)
    dominant = kernel_of_path(wl.layers[0][2].plan(M)["path"])
    traffic = lookup_traffic(dominant, args.workload, M)
    avg_launch_us = round(1e3 * float(np.mean(per_fwd_eff)), 3)
    if M > 16:
        # a dense contraction: 2*M*N*K flops per forward against the bf16 tensor peak
        flops_per_fwd = [2.0 * M * spec.N * spec.K for _, spec, _ in wl.layers]
        tflops = sum(flops_per_fwd) / (sum(per_fwd_eff) * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(tflops / peaks["bf16_tflops"], 4), "traffic": traffic,
                    "kernel": dominant, "peak_source": f"{peak_src} bf16_tflops (burst)",
                    "frac_of_sustained": round(tflops / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), 4),
                    "avg_launch_us": avg_launch_us, "launch_time_from": launch_source,
                    "event_node_us": round(1e3 * float(np.mean(per_fwd)), 3),
                    "algorithmic_flops_per_launch": int(np.mean(flops_per_fwd))}
    else:
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                    "kernel": dominant, "peak_source": f"{peak_src} hbm_gbs",
                    "avg_launch_us": avg_launch_us, "launch_time_from": launch_source,
                    "launches_per_forward": launches_per_fwd[0],
                    "event_node_us": round(1e3 * float(np.mean(per_fwd)), 3),
                    "algorithmic_bytes_per_launch": int(np.mean(bytes_per_fwd))}

    # ------------------------------------------------ end to end through the public API
    e2e_ms, h2d, d2h = time_e2e(wl, M, min(args.steps, 200), 3)
    e2e = {"value": round(1e3 * statistics.fmean(e2e_ms) / layers, 3), "unit": "us/layer",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "how": "per step: pinned-host x -> device copy, the forwards as eager C-ABI calls one after another "
                  "on one stream, y -> pinned host; timed by CUDA events on that stream"}

    out = {
        "metric": METRIC, "value": round(us_per_layer, 3), "unit": "us/layer", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "timing": {"regions": args.regions, "steps_per_region": args.steps,
                   "region_ms_per_step": [round(v / args.steps, 5) for v in region_ms],
                   "spread": round((max(region_ms) - min(region_ms)) / statistics.median(region_ms), 4),
                   "warmup": f"{args.warmup} steps, then whole weight-copy cycles until {WARMUP_SECONDS} s of "
                             "replays; value = the median region"},
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; uniform indices, N(0,1) codebooks and activations, lognormal scales)",
        "config": {"workload": args.workload, "M": M, "layers_per_step": layers,
                   "shapes": [[spec.N, spec.K] for _, spec, _ in wl.layers[:7]],
                   "format": "rvq12_4 block-64" if args.workload != "vq16-4096-rht" else "vq16 per-row",
                   "parallelism": f"replicas x{world}",
                   "l2": L2_NOTE.format(r=R, mb=R * wl.weight_bytes() / 1e6) + (
                       "; the 65,536-entry codebook is one table shared by the copies (L2-resident)"
                       if wl.layers[0][1].fmt in _16BIT else ""),
                   "layer": ("MLP step / 3 weight matrices: gate and up (same x) run concurrently on two "
                             "streams, half of the SMs each (vq_linear_set_sm_budget), then down"
                             if wl.concurrent_gate_up else "one vq_linear_forward (one weight matrix)"),
                   "hbm_gbs": round(sum(bytes_per_fwd) / (ms_per_step * 1e-3) / 1e9, 1)},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": int(wl.launches_per_step(M) * args.steps),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload, M, budget_s=args.cpu_seconds)
    if rank == 0 and not args.no_detail:
        out["detail"] = detail(args, peaks, wl, gpu_index=smi_index)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank value over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_over_ranks(total_ms_local: float, steps: int, layers_per_step: int, world: int):
    """Whole-job timing: the slowest rank's time; every rank ran `layers_per_step` layers per step.

    Returns (ms_per_step, us_per_layer) where us_per_layer divides by the layers all ranks ran.
    """
    total_ms = max_over_ranks(total_ms_local, world)
    ms_per_step = total_ms / steps
    return ms_per_step, 1e3 * ms_per_step / (layers_per_step * world)



def kernel_of_path(path):
    import compressed_index_matmul_b200 as vq

    return {vq.VQ_PATH_LUT: "lut_gemv_kernel", vq.VQ_PATH_GATHER: "vq16_gemv_kernel",
            vq.VQ_PATH_GEMV: "gemv_kernel", vq.VQ_PATH_TC: "tc_gemm_kernel"}[path]


KERNEL_UNITS = {"lut_gemv_kernel": "lut_gemv.cu", "vq16_gemv_kernel": "vq16_gemv.cu", "tc_gemm_kernel": "tc_gemm.cu",
                "gemv_kernel": "gemv.cu"}


def lookup_traffic(kernel, workload, M):
    """DRAM bytes per launch from a committed ncu capture, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
    except ValueError:
        return None
    e = d.get(f"{kernel}|{workload}|M={M}")
    if not e:
        return None
    from compressed_index_matmul_b200.build import source_digest

    # the digest of the kernel's own translation unit, every header and the flags
    if e.get("source_digest") != source_digest(KERNEL_UNITS.get(kernel)):
        return None
    return e.get("dram_bytes_per_launch")


def detail(args, peaks, main_wl, gpu_index=None):
    """The rest of the metric: the other batch sizes of the headline workload and every
    other workload at each of its M, the rotations and the encoder.  The compute-bound
    prefill rows come first (before the GPU has run minutes of other work, which can put
    it under its power cap); every row carries the clocks sampled while it was timed."""
    steps = max(10, min(args.steps, 300))
    res = {}
    if args.workload != "prefill-8192":
        try:
            wl = Workload("prefill-8192", max_M=1024)
            for M in (64, 256, 1024):
                r = measure(wl, M, max(20, steps // 4), 3, peaks, with_kernels=False, gpu_index=gpu_index)
                r["tensor_frac"] = r["tflops"] / peaks["bf16_tflops"]
                r["tensor_frac_sustained"] = r["tflops"] / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
                res[f"prefill-8192 M={M}"] = r
            del wl
        except Exception as exc:  # the tensor-core path reports why it could not run
            res["prefill-8192"] = {"error": str(exc)[:300]}
    for M in (4, 16):
        res[f"{args.workload} M={M}"] = measure(main_wl, M, steps, 3, peaks, gpu_index=gpu_index)
    for name, Ms in (("single-256", (1,)), ("smollm-135m-stack", (1, 4, 16)), ("vq16-4096-rht", (1, 8)),
                     ("llama3-8b-mlp-corr", (1, 16))):
        if name == args.workload:
            continue
        wl = Workload(name, max_M=16)
        for M in Ms:
            r = measure(wl, M, steps, 3, peaks, with_kernels=(name != "smollm-135m-stack"), gpu_index=gpu_index)
            if name == "smollm-135m-stack":
                r["us_per_transformer_layer"] = 1e3 * r["ms_per_step"] / 30
            res[f"{name} M={M}"] = r
        del wl
    for M in (1, 8):
        res[f"rotation 4096 M={M}"] = time_rotations(4096, M, steps)
        for label, shards in (("qkv 4096+1024+1024", (4096, 1024, 1024)), ("gate-up 14336+14336", (14336, 14336))):
            res[f"sharded output rotation {label} M={M}"] = time_sharded_rotation(shards, M, steps)
    for bpw in (3, 4, 5):  # the residual ladder
        name = f"vq16-ladder-4096-{bpw}bpw"
        if name == args.workload:
            continue
        wl = Workload(name, max_M=8)
        for M in (1, 8):
            res[f"{name} M={M}"] = measure(wl, M, steps, 3, peaks, gpu_index=gpu_index)
        del wl
    from synth import FMT_RVQ12_4
    for fmt, sg, label in ((FMT_RVQ12_4, 64, "rvq12_4 block-64"), (FMT_VQ16, 4096, "vq16 per-row")):
        res[f"encode 4096x4096 {label}"] = time_encoder(LayerSpec(4096, 4096, fmt, sg))
    for v in res.values():
        for k in list(v):
            if isinstance(v[k], float):
                v[k] = round(v[k], 4)
    return res


def time_sharded_rotation(shards, M, steps):
    """Device time per launch of the shard-batched output rotation (vq_rht_apply_output_sharded):
    every column shard of an [M, sum(shards)] fp16 output rotated with its own signs."""
    import torch

    import compressed_index_matmul_b200 as vq

    N = int(sum(shards))
    y = torch.from_numpy(make_x(M, N, DT_F16, cfg_id=3).view(np.int16)).cuda().view(torch.float16)
    sg = torch.from_numpy(make_signs(N, cfg_id=3)).cuda()
    out = torch.empty_like(y)
    stream = torch.cuda.Stream()
    reps = 20
    with torch.cuda.stream(stream):
        vq.vq_rht_apply_output_sharded(y, out, sg, M, N, shards, DT_F16, stream.cuda_stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                vq.vq_rht_apply_output_sharded(y, out, sg, M, N, shards, DT_F16, stream.cuda_stream)
        g.replay()
        stream.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(max(1, steps // reps)):
            g.replay()
        t1.record(stream)
    torch.cuda.synchronize()
    us = 1e3 * t0.elapsed_time(t1) / (reps * max(1, steps // reps))
    return {"M": M, "shards": list(shards), "us_per_launch": us, "launches": 1}


def time_encoder(spec, calls=5):
    """Device time of one nearest-entry encode (vq_encode) of a dense binary32 N x K matrix into
    the planes of `spec` (an encoder runs once per layer, off the forward path)."""
    import torch

    import compressed_index_matmul_b200 as vq

    layer = make_layer(spec, cfg_id=143, tensor_id=spec.fmt)
    N, K, G = spec.N, spec.K, spec.K // 8
    w = (torch.randn((N, K), generator=torch.Generator().manual_seed(143), dtype=torch.float32) * 0.02).cuda()
    out = {}
    if spec.fmt == FMT_VQ16:
        out["idx16"] = torch.zeros(N * G, dtype=torch.int16, device="cuda")
    else:
        out["lo"] = torch.zeros(N * G, dtype=torch.uint8, device="cuda")
        out["hi4"] = torch.zeros(N * G // 2, dtype=torch.uint8, device="cuda")
        if "cb2" in layer:
            out["s2"] = torch.zeros(N * G // 2, dtype=torch.uint8, device="cuda")

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    cb1, cb2 = dev(layer["cb1"]), (dev(layer["cb2"]) if "cb2" in layer else None)
    sc = dev(layer["scales"])
    cbs = vq.make_codebooks(cb1, cb2)

    def once():
        vq.vq_encode(N, K, spec.fmt, spec.scale_group, w, sc, cbs, out.get("lo"), out.get("hi4"), out.get("s2"),
                     out.get("idx16"))

    once()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(calls + 1)]
    evs[0].record()
    for i in range(calls):
        once()
        evs[i + 1].record()
    torch.cuda.synchronize()
    ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(calls)]
    med = statistics.median(ms)
    entries = 65536 if spec.fmt == FMT_VQ16 else 4096 + (16 if "cb2" in layer else 0)
    return {"N": N, "K": K, "ms_per_encode": med, "groups_per_s": N * G / (med * 1e-3),
            "distances_per_s": N * G * entries / (med * 1e-3), "calls": calls}


def time_rotations(K, M, steps):
    """Device time per launch of the standalone input rotation (vq_rht_apply) and the
    output rotation (vq_rht_apply_output) on M rows of K fp16 values, as CUDA graphs."""
    import torch

    import compressed_index_matmul_b200 as vq

    x = torch.from_numpy(make_x(M, K, DT_F16, cfg_id=3).view(np.int16)).cuda().view(torch.float16)
    sg = torch.from_numpy(make_signs(K, cfg_id=3)).cuda()
    out = torch.empty_like(x)
    res = {"M": M, "K": K}
    for name, fn in (("input_us", vq.vq_rht_apply), ("output_us", vq.vq_rht_apply_output)):
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            fn(x, out, sg, M, K, DT_F16, stream.cuda_stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(20):
                    fn(x, out, sg, M, K, DT_F16, stream.cuda_stream)
            g.replay()
            stream.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(max(1, steps // 20)):
                g.replay()
            t1.record(stream)
        torch.cuda.synchronize()
        res[name] = 1e3 * t0.elapsed_time(t1) / (20 * max(1, steps // 20))
    return res


# --------------------------------------------------------------------------- CPU oracle

def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # not Linux
        return os.cpu_count() or 1


_POOLS = {}


def _oracle_rows(orc, layer, x, act, rows, threads):
    """The oracle on rows 0..rows-1 of the full layer, split over `threads` threads
    (ctypes releases the GIL during the C call, so the row subsets run in parallel; the
    thread pool is made once per thread count)."""
    import concurrent.futures as cf

    parts = [p for p in np.array_split(np.arange(rows, dtype=np.int32), threads) if len(p)]
    if len(parts) == 1:
        orc.forward(layer, x, act, rows=parts[0])
        return
    ex = _POOLS.get(threads)
    if ex is None:
        ex = _POOLS[threads] = cf.ThreadPoolExecutor(threads)
    list(ex.map(lambda r: orc.forward(layer, x, act, rows=r), parts))


def cpu_baseline(workload, M, budget_s=15.0, threads=None):
    """Time the oracle on a bounded row sample of each tensor of the workload (rows of
    the full layer, computed exactly as for a whole layer), on `threads` host threads
    (default: every core this process may use); scale to whole layers."""
    from oracle import oracle as orc

    orc.build()
    threads = threads or _host_cores()
    w = WORKLOADS[workload]
    cfg = w["config"] if "config" in w else CONFIGS[w["cfg"]]
    tensors = cfg["tensors"]
    x_cache = {}
    per_layer_s, single_s = [], []
    t_start = time.perf_counter()
    sample_desc = []
    for ti, (label, spec) in enumerate(tensors):
        layer = make_layer(spec, cfg_id=w["cfg"], layer=0, tensor_id=ti)
        if spec.K not in x_cache:
            x_cache[spec.K] = make_x(M, spec.K, cfg["act"], cfg_id=w["cfg"])
        if ti == 0:  # untimed: loads the oracle library and starts the threads once
            _oracle_rows(orc, layer, x_cache[spec.K], cfg["act"], min(spec.N, threads), threads)
        rows = max(8, min(spec.N, int(threads * 2048 * 4096 / spec.K)))
        # shrink the sample until one tensor fits its share of the budget
        while True:
            t0 = time.perf_counter()
            _oracle_rows(orc, layer, x_cache[spec.K], cfg["act"], rows, threads)
            dt = time.perf_counter() - t0
            if dt * spec.N / rows < 4 * budget_s or rows <= 8:
                break
            rows = max(8, rows // 4)
        per_layer_s.append(dt * spec.N / rows)
        # the same oracle on one thread, on a 1/threads share of the sample (about the same wall time)
        rows1 = max(8, rows // threads)
        t0 = time.perf_counter()
        _oracle_rows(orc, layer, x_cache[spec.K], cfg["act"], rows1, 1)
        single_s.append((time.perf_counter() - t0) * spec.N / rows1)
        sample_desc.append(f"{label}: {rows}/{spec.N} rows ({rows1} on one thread)")
        if time.perf_counter() - t_start > budget_s:
            break
    us = 1e6 * float(np.mean(per_layer_s))
    return {"value": round(us, 1), "unit": "us/layer", "cores": threads, "kind": "oracle",
            "single_thread_value": round(1e6 * float(np.mean(single_s)), 1),
            "sample": f"M={M}; " + ", ".join(sample_desc) + f"; {threads} threads over row subsets "
                      "(single_thread_value: one thread); time scaled by N/rows (rows are independent)"}


REFERENCE_SECONDS = 150.0  # the whole --impl reference run, warm-up included


def reference_arm(args):
    """--impl reference: the oracle on the host cores, same workload/metric; rank 0 only.

    Each of the W + K steps times the oracle on a row sample of one tensor of the
    workload (the tensors in turn), sized so that the whole run takes about
    REFERENCE_SECONDS; a step's result is its sample time scaled to the whole tensor
    (rows are independent) and the line reports the mean over the K timed steps."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as orc

    orc.build()
    threads = _host_cores()
    w = WORKLOADS[args.workload]
    cfg = _workload_config(args.workload)
    layers, xs = [], {}
    for ti, (label, spec) in enumerate(cfg["tensors"]):
        layers.append((label, spec, make_layer(spec, cfg_id=w["cfg"], layer=0, tensor_id=ti)))
        if spec.K not in xs:
            xs[spec.K] = make_x(args.batch, spec.K, cfg["act"], cfg_id=w["cfg"])
    # calibration (untimed): seconds per row of each tensor on all threads
    row_s = []
    for label, spec, layer in layers:
        r0 = min(spec.N, 64 * threads)
        _oracle_rows(orc, layer, xs[spec.K], cfg["act"], r0, threads)
        t0 = time.perf_counter()
        _oracle_rows(orc, layer, xs[spec.K], cfg["act"], r0, threads)
        row_s.append(max(1e-9, (time.perf_counter() - t0) / r0))
    per_step = REFERENCE_SECONDS / max(1, args.steps + args.warmup)
    per_layer, rows_used = [], set()
    for k in range(args.warmup + args.steps):
        ti = k % len(layers)
        label, spec, layer = layers[ti]
        rows = int(max(8, min(spec.N, per_step / row_s[ti])))
        t0 = time.perf_counter()
        _oracle_rows(orc, layer, xs[spec.K], cfg["act"], rows, threads)
        dt = time.perf_counter() - t0
        if k >= args.warmup:
            per_layer.append(1e6 * dt * spec.N / rows)
            rows_used.add((label, rows, spec.N))
    v = float(np.mean(per_layer))
    sample = (f"M={args.batch}; each step one tensor in turn, rows 0..r-1 of the full layer on {threads} threads, "
              "time scaled by N/r (rows are independent): " +
              ", ".join(f"{lb} {r}/{n} rows" for lb, r, n in sorted(rows_used)))
    out = {"metric": METRIC, "value": round(v, 1), "unit": "us/layer", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(v * 1e-3 * len(cfg["tensors"]), 3),
           "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded)", "impl": "reference",
           "config": {"workload": args.workload, "M": args.batch, "layer": "one weight matrix"},
           "cpu_baseline": {"value": round(v, 1), "unit": "us/layer", "cores": threads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(v, 1), "unit": "us/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3-8b-mlp")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--no-detail", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--regions", type=int, default=REGIONS,
                    help="timed regions of exactly K steps each (the line reports their median)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
