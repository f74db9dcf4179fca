#!/usr/bin/env python
"""Benchmark of the GQE prefill layer on B200; rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole GQE prefill layer (router, dispatch and
grouped query projection, K/V projection, routed + shared attention, weighted
slot and W_O) over one batch of the workload, issued through the library's C
ABI, captured once as a CUDA graph and replayed. Timing: CUDA events on the
launching stream around every step, L2 flushed before each timed step (256 MiB
written, then 256 MiB read, so no dirty lines are left), max over ranks. Under torchrun
every rank runs an independent replica of the workload (weak scaling, no
data-path collective).

--impl reference times the fp64 CPU oracle (the reference of this build) on
the same workload, on the host cores of rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "GQE prefill layer tokens/s and attn tensor-pipe % of bf16 peak vs seq len"
WORKLOADS = {
    "seq2k": synth.SEQ2K,
    "b4x8k": synth.BATCH4_8K,
    "seq32k": synth.SEQ32K,
    "seq256k": synth.SEQ256K,
    "seq1m": synth.SEQ1M,
    "seq64k": synth.LayerShape(B=1, T=65536, d_model=1024, G=8, M=2, k=1, d_head=64),
    "pool4_k1": synth.POOL4_K1,
    "pool4_k2": synth.POOL4_K2,
}
HEADLINE = "seq2k"
SWEEP = ["b4x8k", "seq32k", "seq256k", "seq1m"]
DISPATCH_TILE, FUSED_SCAN_MAX = 256, 16384  # tokens per dispatch tile; N * tiles for one scan+scatter launch


def launches(s: synth.LayerShape) -> dict:
    """Kernels of this library launched per call of one step."""
    tiles = s.B * -(-s.T // DISPATCH_TILE)
    fused = s.N * tiles <= FUSED_SCAN_MAX
    # dispatch: masks+counts, scan+scatter (one launch or two), the grouped Q GEMM
    # output: the W_O GEMM, with the weighted slot fused in when d_head = 64
    return {"router": 1, "dispatch": 3 if fused else 4, "kv": 1, "attention": 1,
            "output": 1 if s.d_head == 64 else 2}


SHORT_BATCH_ROWS = 4096  # the library's short-batch path: B*T rows at most, d_head 64


def layer_launches(s: synth.LayerShape) -> int:
    """Kernels of this library per gqe_layer_fwd call. Long batches: the step
    calls' kernels, with the shared-head query projection as its own GEMM on
    the side stream instead of tiles of the routed Q GEMM. Short batches
    (B*T <= 4096, d_head 64): router, shared-head Q GEMM, the projections
    (one fused K/V/Q GEMM when M = 2, else a K/V GEMM and an every-expert Q
    GEMM), attention and W_O -- no token-list kernels."""
    if s.B * s.T <= SHORT_BATCH_ROWS and s.d_head == 64:
        return 1 + 1 + (1 if s.M == 2 else 2) + 1 + launches(s)["output"]
    return sum(launches(s).values()) + 1


FLUSH_BYTES = 256 << 20
PAGES_SPEEDUP = {"2k": 1.15, "4k..1024k": "1.67-1.80", "1024k": 1.80,
                 "hardware": "not stated"}


def describe(s: synth.LayerShape) -> str:
    return (f"GQE prefill layer B={s.B} T={s.T} d_model={s.d_model} G={s.G} M={s.M} k={s.k} "
            f"d_head={s.d_head} (+1 shared head)")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "hbm": p["hbm_gbs"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


def flops(s: synth.LayerShape, dense: bool = False):
    """Algorithmic FLOPs per layer pass (active work only)."""
    heads = s.N if dense else s.k * s.G + 1
    slots = s.N if dense else s.n_slots
    R, d, dh = s.R, s.d_model, s.d_head
    attn = 4.0 * dh * heads * s.B * s.T * (s.T + 1) / 2
    return {"attention": attn, "q": 2.0 * R * d * dh * heads, "kv": 4.0 * R * d * dh * s.G,
            "wo": 2.0 * R * slots * dh * d, "router": 0.0 if dense else 2.0 * R * d * s.N}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting"}

    def __init__(self, torch_dev: int, period_s: float = 0.002):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.max_mhz = None

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            self.reasons |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
            if not self.samples:
                self._sample()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b]}


# ---------------------------------------------------------------- GPU arm
class Layer:
    """Device buffers of one layer instance and the C-ABI calls of one step."""

    def __init__(self, rsq, shape: synth.LayerShape, d: dict):
        import torch
        self.rsq, self.s, self.d = rsq, shape, d
        s = shape
        B, T, G, M, k, dh, R, N = s.B, s.T, s.G, s.M, s.k, s.d_head, s.R, s.N
        dev = torch.device("cuda")
        self.cfg = rsq.GQEConfig.of(s)
        # The attention scratch is zero-filled once; every call leaves its
        # split-KV counters zero, so the calls skip clearing them.
        self.cfg_clean = rsq.GQEConfig.of(s, rsq.GQE_FLAG_WS_CLEAN)
        e = torch.empty
        self.idx = e(R, G, k, dtype=torch.int32, device=dev)
        self.r = e(R, G, k, dtype=torch.float32, device=dev)
        self.omega = e(R, G, k, dtype=torch.float32, device=dev)
        self.counts = e(N * B, dtype=torch.int32, device=dev)
        self.offsets = e(N * B + 1, dtype=torch.int32, device=dev)
        self.tok = e(k * G * R, dtype=torch.int32, device=dev)
        self.slot_pos = e(R, G, k, dtype=torch.int32, device=dev)
        self.Qv = e(B, G, k, T, dh, dtype=torch.bfloat16, device=dev)
        self.Qs = e(B, T, dh, dtype=torch.bfloat16, device=dev)
        self.K = e(B, G, T, dh, dtype=torch.bfloat16, device=dev)
        self.V = e(B, G, T, dh, dtype=torch.bfloat16, device=dev)
        self.slots = e(R, s.n_slots * dh, dtype=torch.bfloat16, device=dev)
        self.y = e(R, s.d_model, dtype=torch.bfloat16, device=dev)
        self.wsd = e(rsq.gqe_workspace_bytes(self.cfg, rsq.GQE_WS_DISPATCH), dtype=torch.uint8, device=dev)
        self.wsa = torch.zeros(rsq.gqe_workspace_bytes(self.cfg, rsq.GQE_WS_ATTENTION), dtype=torch.uint8,
                               device=dev)

    def router(self):
        d = self.d
        self.rsq.gqe_router_topk(self.cfg, d["x"], d["W_r"], d["b_r"], self.idx, self.r, self.omega)

    def dispatch(self):
        d = self.d
        self.rsq.gqe_dispatch(self.cfg, self.idx, d["x"], d["W_q"], d["W_qs"], self.counts,
                              self.offsets, self.tok, self.slot_pos, self.Qv, self.Qs, self.wsd)

    def kv(self):
        d = self.d
        self.rsq.gqe_kv_proj(self.cfg, d["x"], d["W_k"], d["W_v"], self.K, self.V)

    def attention(self):
        self.rsq.gqe_attention_fwd(self.cfg_clean, self.Qv, self.Qs, self.K, self.V, self.slots, self.wsa)

    def attention_expert_major_fn(self):
        """The same attention over compacted expert-major tiles (the routed
        queries rewritten in token-list order once, outside any timing)."""
        import torch
        rsq, s, d = self.rsq, self.s, self.d
        cfg = rsq.GQEConfig.of(s, rsq.GQE_FLAG_EXPERT_MAJOR)
        Qe = torch.empty(s.k * s.G * s.R, s.d_head, dtype=torch.bfloat16, device="cuda")
        Qs = torch.empty_like(self.Qs)
        rsq.gqe_dispatch(cfg, self.idx, d["x"], d["W_q"], d["W_qs"], self.counts, self.offsets,
                         self.tok, self.slot_pos, Qe, Qs, self.wsd)
        slots = torch.zeros_like(self.slots)

        def f():
            rsq.gqe_attention_fwd_compact(cfg, Qe, Qs, self.K, self.V, self.idx, self.offsets,
                                          self.tok, slots)
        return f

    def output(self):
        self.rsq.gqe_output_proj(self.cfg, self.slots, self.omega, self.d["W_o"], self.y)

    CALLS = ("router", "dispatch", "kv", "attention", "output")


def device_inputs_from_synth(inp: synth.LayerInputs) -> dict:
    import torch

    def b16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    d = {"x": b16(inp.x), "W_r": torch.from_numpy(inp.W_r).cuda(),
         "b_r": None if inp.b_r is None else torch.from_numpy(inp.b_r).cuda(),
         "W_q": b16(inp.W_q), "W_qs": b16(inp.W_qs), "W_k": b16(inp.W_k), "W_v": b16(inp.W_v),
         "W_o": b16(inp.W_o), "W_o_dense": b16(inp.W_o_dense)}
    return d


def device_inputs_seeded(shape: synth.LayerShape, seed: int) -> dict:
    """Same recipe as synth (x ~ N(0,1), weights ~ N(0, 1/d)), drawn on the
    device with torch's seeded generator (for sizes too large to draw on the
    host quickly)."""
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    s, sd = shape, shape.d_model ** -0.5
    d = {"x": torch.randn(s.R, s.d_model, device="cuda", generator=g).to(torch.bfloat16),
         "W_r": torch.randn(s.d_model, s.N, device="cuda", generator=g) * sd, "b_r": None}
    for nm, shp in (("W_q", (s.d_model, s.N * s.d_head)), ("W_qs", (s.d_model, s.d_head)),
                    ("W_k", (s.d_model, s.G * s.d_head)), ("W_v", (s.d_model, s.G * s.d_head)),
                    ("W_o", (s.n_slots * s.d_head, s.d_model)),
                    ("W_o_dense", (s.N * s.d_head, s.d_model))):
        d[nm] = (torch.randn(*shp, device="cuda", generator=g) * sd).to(torch.bfloat16)
    return d


def _graph(f):
    """f captured once as a CUDA graph (on a side stream; warm calls made before),
    or None where capture is not possible: replays then time device work only,
    with no host issue time between the kernels of a step."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            f()
        torch.cuda.current_stream().wait_stream(s)
        return g
    except Exception:  # noqa: BLE001 - capture unavailable: eager calls
        torch.cuda.synchronize()
        return None


def time_steps(layer: Layer, steps: int, warmup: int, flush, sync_ranks) -> dict:
    """Times `steps` layer passes call by call (each entry point captured as its
    own CUDA graph and replayed, events between them); returns total ms and
    per-call ms sums."""
    import torch
    for _ in range(warmup):
        for c in Layer.CALLS:
            getattr(layer, c)()
    torch.cuda.synchronize()
    graphs = {c: _graph(getattr(layer, c)) for c in Layer.CALLS}
    run = {c: (graphs[c].replay if graphs[c] is not None else getattr(layer, c)) for c in Layer.CALLS}
    for _ in range(2):
        for c in Layer.CALLS:
            run[c]()
    torch.cuda.synchronize()
    n = len(Layer.CALLS)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    sync_ranks()
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record()
        for j, c in enumerate(Layer.CALLS):
            run[c]()
            ev[i][j + 1].record()
    torch.cuda.synchronize()
    sync_ranks()
    per = {c: 0.0 for c in Layer.CALLS}
    total = 0.0
    for i in range(steps):
        total += ev[i][0].elapsed_time(ev[i][n])
        for j, c in enumerate(Layer.CALLS):
            per[c] += ev[i][j].elapsed_time(ev[i][j + 1])
    return {"total_ms": total, "per_call_ms": per, "graphs": all(g is not None for g in graphs.values())}


def time_layer(rsq, shape, d, steps, warmup, flush, sync_ranks=lambda: None, eager: bool = False) -> float:
    """Total ms of `steps` passes of the whole layer through its one entry
    point, gqe_layer_fwd (device time per step; L2 flushed before each when
    `flush` is given), replayed from a CUDA graph unless `eager`."""
    import torch
    cfg = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_WS_CLEAN)
    ws = torch.zeros(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_LAYER), dtype=torch.uint8, device="cuda")
    y = torch.empty(shape.R, shape.d_model, dtype=torch.bfloat16, device="cuda")

    def f():
        rsq.gqe_layer_fwd(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                          d["W_o"], y, ws)

    return _time_calls(f, steps, warmup, flush, sync_ranks, eager)


def _time_calls(f, steps, warmup, flush, sync_ranks=lambda: None, eager: bool = False) -> float:
    import torch
    for _ in range(warmup):
        f()
    torch.cuda.synchronize()
    if not eager:
        g = _graph(f)
        if g is not None:
            f = g.replay
            for _ in range(2):
                f()
            torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    sync_ranks()
    torch.cuda.synchronize()
    for a, b in ev:
        if flush is not None:
            flush()
        a.record()
        f()
        b.record()
    torch.cuda.synchronize()
    sync_ranks()
    return sum(a.elapsed_time(b) for a, b in ev)


def time_dense(rsq, shape, d, steps, warmup, flush, eager: bool = False) -> float:
    import torch
    cfg = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_WS_CLEAN)
    ws = torch.zeros(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DENSE), dtype=torch.uint8, device="cuda")
    y = torch.empty(shape.R, shape.d_model, dtype=torch.bfloat16, device="cuda")

    def f():
        rsq.gqa_dense_fwd(cfg, d["x"], d["W_q"], d["W_k"], d["W_v"], d["W_o_dense"], y, ws)

    return _time_calls(f, steps, warmup, flush, eager=eager)


def gpu_local_cpus() -> set | None:
    """The host CPUs that NVML reports as local to the current GPU (its NUMA
    node), intersected with the ones this process may run on; None if NVML
    or the query is unavailable. A read-only query."""
    import torch
    try:
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(torch.cuda.current_device())
        uuid = str(getattr(props, "uuid", ""))
        h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid if not uuid.startswith("GPU-") else uuid).encode())
        words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        local = {64 * i + bit for i, w in enumerate(words) for bit in range(64) if (int(w) >> bit) & 1}
        cpus = local & os.sched_getaffinity(0)
        return cpus or None
    except Exception:  # noqa: BLE001 - no NVML, no binding
        return None


def time_e2e(rsq, shape, d, steps, warmup) -> dict:
    """gqe_layer_fwd with x copied in from pinned host memory and y copied
    back, every step, inside the timed region, pipelined: stage i copies in
    the input of step i+1, runs the layer of step i and copies out the result
    of step i-1, as three independent branches (two device buffers each).
    Each stage is captured once as a CUDA graph (one per buffer parity) and
    replayed, so the host issues one launch per step; if capture is not
    possible the same stages run eagerly."""
    import torch
    # The pinned host buffers are placed on the GPU's own NUMA node: this
    # thread runs on the CPUs local to the GPU while it allocates and drives
    # the copies (the previous affinity is restored afterwards).
    saved = os.sched_getaffinity(0)
    local = gpu_local_cpus()
    if local is not None:
        os.sched_setaffinity(0, local)
    try:
        return _time_e2e(rsq, shape, d, steps, warmup, local)
    finally:
        os.sched_setaffinity(0, saved)


def _time_e2e(rsq, shape, d, steps, warmup, local) -> dict:
    import torch
    cfg = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_WS_CLEAN)
    ws = torch.zeros(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_LAYER), dtype=torch.uint8, device="cuda")
    x_h = d["x"].cpu().pin_memory()
    y_h = torch.empty(shape.R, shape.d_model, dtype=torch.bfloat16).pin_memory()
    x_d = [torch.empty_like(d["x"]) for _ in range(2)]
    y_d = [torch.empty(shape.R, shape.d_model, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    main = torch.cuda.Stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def stage(j):  # enqueued on the current stream
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        with torch.cuda.stream(s_in):
            x_d[1 - j].copy_(x_h, non_blocking=True)  # input of the next step
        with torch.cuda.stream(s_out):
            y_h.copy_(y_d[1 - j], non_blocking=True)  # result of the previous step
        rsq.gqe_layer_fwd(cfg, x_d[j], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                          d["W_o"], y_d[j], ws, stream=cur)
        cur.wait_stream(s_in)
        cur.wait_stream(s_out)

    with torch.cuda.stream(main):
        for i in range(max(2, warmup)):
            stage(i % 2)
    torch.cuda.synchronize()
    graphs = None
    try:
        gs = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
        for j in (0, 1):
            with torch.cuda.graph(gs[j], stream=main):
                stage(j)
        with torch.cuda.stream(main):
            for i in range(2):
                gs[i % 2].replay()
        torch.cuda.synchronize()
        graphs = gs
    except Exception:  # noqa: BLE001 - capture unavailable: eager stages
        torch.cuda.synchronize()
        graphs = None
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(main):
        a.record(main)
        x_d[0].copy_(x_h, non_blocking=True)  # input of step 0
        for i in range(steps):
            if graphs is not None:
                graphs[i % 2].replay()
            else:
                stage(i % 2)
        y_h.copy_(y_d[(steps - 1) % 2], non_blocking=True)  # result of the last step
        b.record(main)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    return {"ms": ms, "h2d": x_h.numel() * 2, "d2h": y_h.numel() * 2,
            "graph": graphs is not None, "host_cpus": len(local) if local is not None else None}


def roofline_of(shape, per_call_ms: dict, steps: int, pk: dict, traffic=None):
    fl = flops(shape)
    s = shape
    units = {
        "attention": ("tensor", fl["attention"] / 1e12, "TFLOP/s", pk["bf16"]),
        "kv": ("tensor", fl["kv"] / 1e12, "TFLOP/s", pk["bf16"]),
        "output": ("tensor", fl["wo"] / 1e12, "TFLOP/s", pk["bf16"]),
        "dispatch": ("tensor", fl["q"] / 1e12, "TFLOP/s", pk["bf16"]),
        "router": ("hbm", (s.R * s.d_model * 2 + s.d_model * s.N * 4 + s.R * s.G * s.k * 12) / 1e9,
                   "GB/s", pk["hbm"]),
    }
    # The attention kernel: the path's dominant single kernel at every
    # measured length (the dispatch call is three kernels), and the one the
    # method changes.
    top = "attention"
    bound, work, unit, peak = units[top]
    avg_s = per_call_ms[top] / steps / 1e3
    ach = work / avg_s if avg_s > 0 else 0.0
    return {"kernel": top, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
            "frac": ach / peak, "peak_source": f"{pk['source']} burst", "traffic": traffic,
            "avg_launch_ms": avg_s * 1e3}


def router_bytes(s: synth.LayerShape) -> float:
    """Algorithmic HBM bytes of the router: x read once, W_r, idx/r/omega written."""
    return s.R * s.d_model * 2 + s.d_model * s.N * 4 + s.R * s.G * s.k * 12


def call_fractions(s: synth.LayerShape, per_call_ms: dict, steps: int, pk: dict) -> dict:
    """Each entry point's achieved rate against its roofline (of the measured
    peaks): the router on HBM bytes; the K/V and W_O GEMMs, the dispatch call
    (token-list kernels plus the grouped Q GEMM, FLOPs of the Q GEMM) and the
    attention on bf16 tensor FLOPs (burst peak: each is timed alone)."""
    fl = flops(s)
    t = {c: per_call_ms[c] / steps / 1e3 for c in per_call_ms}
    out = {"router_hbm_frac": router_bytes(s) / t["router"] / 1e9 / pk["hbm"]}
    for call, key in (("kv", "kv"), ("output", "wo"), ("dispatch", "q"), ("attention", "attention")):
        out[f"{call}_tensor_frac"] = fl[key] / t[call] / 1e12 / pk["bf16"]
    return {k: round(v, 4) for k, v in out.items()}


def cpu_baseline(shape: synth.LayerShape, max_tokens: int | None = None,
                 min_seconds: float = 0.0, threads: int | None = None) -> dict:
    """The oracle as it stands, on this host: full layer passes over one
    sequence (the first max_tokens tokens), repeated until min_seconds.
    `threads` limits the BLAS thread pool (None: as many as it has)."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    T = shape.T if max_tokens is None else min(shape.T, max_tokens)
    s = synth.LayerShape(1, T, shape.d_model, shape.G, shape.M, shape.k, shape.d_head)
    inp = synth.make_layer_inputs(s, with_dense=False)
    with threadpool_limits(limits=threads):
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        passes, dt = 0, 0.0
        t0 = time.perf_counter()
        while passes == 0 or (dt < min_seconds and passes < 1000):
            oracle.gqe_layer(inp)
            passes += 1
            dt = time.perf_counter() - t0
    return {"value": T * passes / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} full oracle layer passes over {T} tokens of one sequence "
                      f"(fp64 numpy, {dt:.2f} s, {cores} BLAS threads)", "seconds": dt / passes}


def max_over_ranks(value: float, dist, device) -> float:
    """Largest `value` over all ranks (the job is as slow as its slowest rank)."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (max_ms / 1e3)


def summary_of(out: dict) -> dict:
    """Short per-workload table (the last key of the line): T, B, GQE and
    dense layer ms, speed-up, attention fraction of the bf16 peak, and the
    other calls' fractions of their rooflines."""
    def r4(v):
        return None if v is None else round(float(v), 4)

    rows = [{"workload": out["config"]["workload"].split(":")[0], "gqe_ms": r4(out["ms_per_step"]),
             "dense_ms": r4(out["dense_gqa"]["ms_per_step"]),
             "speedup": r4(out["dense_gqa"]["speedup_gqe_over_dense"]),
             "attn_frac": r4(out["roofline"]["frac"]), **out.get("fractions", {})}]
    for row in out.get("sweep", []):
        rows.append({"workload": row["workload"].split(":")[0], "gqe_ms": r4(row["gqe_ms"]),
                     "dense_ms": r4(row["dense_ms"]), "speedup": r4(row["speedup"]),
                     "attn_frac": r4(row["attn_frac_of_bf16_peak"]), **row.get("fractions", {})})
    for row in out.get("pool_sweep", []):
        rows.append({"workload": row["workload"].split(":")[0], "gqe_ms": r4(row["gqe_ms"]),
                     "dense_ms": r4(row["dense_ms"]), "speedup": r4(row["speedup"]),
                     "attn_frac": r4(row["attn_frac_of_bf16_peak"]),
                     "hot_expert_share": r4(row["hot_expert_share"]), **row.get("fractions", {})})
    return {"per_workload": rows, "peaks": "fractions of the measured peaks (bf16 burst, HBM copy)"}


def run_ours(args, rank: int, world: int, dist):
    import torch
    import routed_sparse_query_b200 as rsq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    pk = peaks()
    shape = WORKLOADS[args.workload]
    inp = synth.make_layer_inputs(shape, seed=synth.DEFAULT_SEED + rank)
    d = device_inputs_from_synth(inp)
    layer = Layer(rsq, shape, d)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    read_buf = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def flush():
        # Write 256 MiB (evicts every input of the step from the 126 MB L2),
        # then read another 256 MiB, so that the dirty lines of the write are
        # written back before the step and L2 holds clean, unrelated lines.
        flush_buf.zero_()
        read_buf.sum()  # float32: one reduction, no widened temporary

    def sync_ranks():
        if dist is not None:
            dist.barrier()

    warmup = max(3, args.warmup)
    with ClockSampler(torch.cuda.current_device()) as clk:
        # The step: one pass of the whole layer through gqe_layer_fwd.
        layer_ms = time_layer(rsq, shape, d, args.steps, warmup, flush, sync_ranks)
        # The same call issued from Python every step (host issue time included).
        eager_ms = time_layer(rsq, shape, d, args.steps, warmup, flush, sync_ranks, eager=True)
        # The same steps call by call, for the per-call times (roofline).
        res = time_steps(layer, args.steps, warmup, flush, sync_ranks)
    if rsq.gqe_read_status() != 0:
        raise RuntimeError("device-side status set during the timed steps")
    max_ms = max_over_ranks(layer_ms, dist, "cuda")
    ms_per_step = max_ms / args.steps
    value = job_throughput(shape.R, world, args.steps, max_ms)

    e2e = time_e2e(rsq, shape, d, args.steps, warmup)
    e2e_value = job_throughput(shape.R, world, args.steps, max_over_ranks(e2e["ms"], dist, "cuda"))

    dense_ms = max_over_ranks(time_dense(rsq, shape, d, args.steps, warmup, flush) / args.steps,
                              dist, "cuda")
    dense_eager_ms = max_over_ranks(time_dense(rsq, shape, d, args.steps, warmup, flush, eager=True) /
                                    args.steps, dist, "cuda")
    eager_ms = max_over_ranks(eager_ms, dist, "cuda") / args.steps
    if dist is not None:
        dist.barrier()
    if rank != 0:
        return None

    traffic = None
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof):
        try:
            with open(prof) as f:
                traffic = json.load(f).get(args.workload)
        except ValueError:
            traffic = None
    roof = roofline_of(shape, res["per_call_ms"], args.steps, pk, traffic)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.workload}: {describe(shape)}", "global_batch": shape.B * world,
                   "seq_len": shape.T, "parallelism": f"replicas{world}",
                   "l2": "flushed before every timed step (256 MiB written, then 256 MiB read)",
                   "timing": "one gqe_layer_fwd call per step, captured once as a CUDA graph and replayed "
                             "(device time; eager_ms_per_step: the call issued from Python every step)",
                   "inputs": "seeded synth recipe: x ~ N(0,1) bf16, weights ~ N(0,1/d_model) bf16, "
                             "router fp32"},
        "gpu_launches": layer_launches(shape) * args.steps,
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "api": "gqe_layer_fwd",
                "host_buffers": (f"pinned, allocated from the {e2e['host_cpus']} CPUs local to the GPU"
                                 if e2e["host_cpus"] else "pinned (GPU-local CPUs unknown)"),
                "pipelining": "copies of steps i+1 (in) and i-1 (out) overlap the layer of step i",
                "cuda_graph_stages": e2e["graph"]},
        "roofline": roof,
        "breakdown_ms_per_step": {c: v / args.steps for c, v in res["per_call_ms"].items()},
        "fractions": call_fractions(shape, res["per_call_ms"], args.steps, pk),
        "breakdown_note": "per entry point, each captured as its own CUDA graph, replayed call by call "
                          "in a second loop of the same steps",
        "eager_ms_per_step": eager_ms,
        "dense_gqa": {"ms_per_step": dense_ms,
                      "tokens_per_s": shape.R * world / (dense_ms / 1e3),
                      "speedup_gqe_over_dense": dense_ms / ms_per_step,
                      "eager_ms_per_step": dense_eager_ms,
                      "eager_speedup": dense_eager_ms / eager_ms},
        "pages_speedup_context": PAGES_SPEEDUP,
    }
    if world == 1 and not args.no_sweep:
        out["sweep"] = sweep(rsq, pk, args)
        out["decode"] = decode_bench(rsq, pk, args.steps)
        if shape.T <= 8192:
            out["backward"] = backward_bench(rsq, shape, d)
    if world == 1 and not args.no_pool:
        out["pool_sweep"] = sweep_pool(rsq, pk, args)
    if world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(shape, min_seconds=10.0)
        one = cpu_baseline(shape, min_seconds=5.0, threads=1)
        out["cpu_baseline"]["one_core"] = {k: one[k] for k in ("value", "unit", "cores", "sample")}
        out["cpu_baseline"]["host_cores"] = os.cpu_count()
    out["summary"] = summary_of(out)
    return out


def backward_flops(shape) -> float:
    """Algorithmic FLOPs of one layer backward (selection fixed; the forward
    recomputation not counted). Attention, per stream and causal (query, key)
    pair: S recomputed, dP = dO V^T, dQ, dK, dV -- five products of 2 dh
    FLOPs. Projections: dS = dy W_O^T and dW_O = S^T dy (2 R d S dh each),
    dx and the weight gradients over the concatenated columns
    [Q of every expert | shared Q | K | V | router] (2 R d C each)."""
    B, T, d, G, M, k, dh = shape.B, shape.T, shape.d_model, shape.G, shape.M, shape.k, shape.d_head
    R, N = B * T, G * M
    streams = B * (G * k + 1)
    attn = 5 * 2 * dh * (T * (T + 1) // 2) * streams
    sdh = (G * k + 2) * dh
    cols = N * dh + dh + 2 * G * dh + N
    return float(attn + 2 * (2 * R * d * sdh) + 2 * (2 * R * d * cols))


def backward_bench(rsq, shape, d, steps: int = 5) -> dict:
    """One gqe_layer_bwd call (forward recomputation included) on the bench
    workload, CUDA-event timed after two warm-up calls; dy ~ N(0, 1)."""
    import torch
    cfg = rsq.GQEConfig.of(shape, rsq.GQE_FLAG_WS_CLEAN)
    ws = torch.zeros(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_BACKWARD), dtype=torch.uint8, device="cuda")
    R, dm, dh, N, G = shape.R, shape.d_model, shape.d_head, shape.N, shape.G
    f32 = lambda *sh: torch.empty(*sh, dtype=torch.float32, device="cuda")  # noqa: E731
    g = torch.Generator(device="cuda").manual_seed(7)
    dy = torch.randn(R, dm, device="cuda", generator=g)
    outs = (f32(R, dm), f32(dm, N), f32(N), f32(dm, N * dh), f32(dm, dh), f32(dm, G * dh), f32(dm, G * dh),
            f32((shape.k * G + 2) * dh, dm))

    def f():
        rsq.gqe_layer_bwd(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"], d["W_o"], dy,
                          *outs, ws)
    for _ in range(2):
        f()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        f()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    fl = backward_flops(shape)
    return {"workload": describe(shape), "ms_per_call": ms, "tokens_per_s": R / (ms / 1e3), "steps": steps,
            "flops": fl, "tflops_excl_forward": fl / (ms / 1e3) / 1e12,
            "path": "forward recomputed (attention keeps each row's log-sum-exp); tcgen05 attention backward "
                    "(dQ per query tile, dK/dV per key tile); projection gradients on the tcgen05 GEMM with an "
                    "fp32 epilogue; router backward through the weighted slot on the CUDA cores"}


DECODE = {"batch": 64, "cache": 32768}  # decode measurement: 64 sequences, 32k cached tokens


def decode_bench(rsq, pk, steps: int) -> dict:
    """One decode step (a new token per sequence against a 32k-token K/V cache)
    through gqe_decode_step and gqa_dense_decode_step, CUDA-event timed. The
    cache and weights are drawn on the device with the synth distributions
    (K, V ~ N(0, 1) like x W with x ~ N(0, 1), W ~ N(0, 1/d))."""
    import torch
    B, T = DECODE["batch"], DECODE["cache"] + 1
    s = synth.LayerShape(B, T, 1024, 8, 2, 1, 64)
    g = torch.Generator(device="cuda").manual_seed(4321)
    d = device_inputs_seeded(synth.LayerShape(B, 1, s.d_model, s.G, s.M, s.k, s.d_head), 4321)
    cap = T
    Kc = torch.randn(B, s.G, cap, s.d_head, device="cuda", generator=g).to(torch.bfloat16)
    Vc = torch.randn(B, s.G, cap, s.d_head, device="cuda", generator=g).to(torch.bfloat16)
    cfg = rsq.GQEConfig.of(s)
    ws = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DECODE), dtype=torch.uint8, device="cuda")
    wsd = torch.empty(rsq.gqe_workspace_bytes(cfg, rsq.GQE_WS_DENSE_DECODE), dtype=torch.uint8,
                      device="cuda")
    y = torch.empty(B, s.d_model, dtype=torch.bfloat16, device="cuda")

    def f():
        rsq.gqe_decode_step(cfg, d["x"], d["W_r"], d["b_r"], d["W_q"], d["W_qs"], d["W_k"], d["W_v"],
                            d["W_o"], Kc, Vc, y, ws)

    def fd():
        rsq.gqa_dense_decode_step(cfg, d["x"], d["W_q"], d["W_k"], d["W_v"], d["W_o_dense"], Kc, Vc,
                                  y, wsd)

    n = max(3, min(steps, 50))
    ms = _time_calls(f, n, 3, None) / n
    dms = _time_calls(fd, n, 3, None) / n
    if rsq.gqe_read_status() != 0:
        raise RuntimeError("device-side status set in the decode measurement")
    kv_bytes = 2 * B * s.G * T * s.d_head * 2  # the cache is read once per step
    return {"workload": f"decode: {B} sequences, {T - 1} cached tokens each, one new token "
                        f"(d_model=1024, G=8, M=2, k=1, d_head=64)",
            "steps": n, "gqe_ms": ms, "gqe_tokens_per_s": B / (ms / 1e3),
            "dense_ms": dms, "dense_tokens_per_s": B / (dms / 1e3), "speedup": dms / ms,
            "kv_cache_bytes": kv_bytes, "kv_gbs": kv_bytes / (ms / 1e3) / 1e9,
            "kv_frac_of_hbm_peak": kv_bytes / (ms / 1e3) / 1e9 / pk["hbm"],
            "l2": "cache (4.3 GB) larger than L2, not flushed"}


def sweep(rsq, pk, args):
    """GQE vs dense GQA at every sequence length of the measured workloads."""
    import torch
    rows = []
    names = SWEEP if args.sweep_max is None else SWEEP[:SWEEP.index(args.sweep_max) + 1]
    for name in names:
        s = WORKLOADS[name]
        d = device_inputs_seeded(s, 1234)
        layer = Layer(rsq, s, d)
        est = flops(s)["attention"] / 0.5e15  # seconds per step at 0.5 PFLOP/s
        steps = max(2, min(args.steps, int(2.0 / max(est, 1e-6))))
        res = time_steps(layer, steps, 2, None, lambda: None)
        dense_ms = time_dense(rsq, s, d, steps, 1, None) / steps
        gq_ms = time_layer(rsq, s, d, steps, 1, None) / steps
        attn_s = res["per_call_ms"]["attention"] / steps / 1e3
        ach = flops(s)["attention"] / attn_s / 1e12
        em_s = _time_calls(layer.attention_expert_major_fn(), steps, 1, None) / steps / 1e3
        rows.append({"workload": f"{name}: {describe(s)}", "T": s.T, "B": s.B, "steps": steps,
                     "gqe_ms": gq_ms, "gqe_tokens_per_s": s.R / (gq_ms / 1e3),
                     "dense_ms": dense_ms, "dense_tokens_per_s": s.R / (dense_ms / 1e3),
                     "speedup": dense_ms / gq_ms, "attn_tflops": ach,
                     "attn_frac_of_bf16_peak": ach / pk["bf16"],
                     "attn_expert_major_ms": em_s * 1e3,
                     "attn_expert_major_frac_of_bf16_peak": flops(s)["attention"] / em_s / 1e12 / pk["bf16"],
                     "l2": "inputs larger than L2, not flushed",
                     "breakdown_ms": {c: v / steps for c, v in res["per_call_ms"].items()},
                     "fractions": call_fractions(s, res["per_call_ms"], steps, pk)})
        if rsq.gqe_read_status() != 0:
            raise RuntimeError(f"device-side status set in sweep {name}")
        del layer, d
        torch.cuda.empty_cache()
    return rows


POOL_SWEEP = [("pool4_k1", True), ("pool4_k2", True), ("pool4_k2", False)]  # (workload, skewed)


def sweep_pool(rsq, pk, args):
    """GQE vs dense GQA on the expert-pool workloads (32 experts, T = 32k):
    k = 1 and 2 with the skew bias (one expert per group takes ~80 % of the
    tokens) and k = 2 balanced. Reports the measured hot-expert share."""
    import torch
    rows = []
    for name, skew in POOL_SWEEP:
        s = WORKLOADS[name]
        d = device_inputs_seeded(s, 1234)
        if skew:
            b = np.zeros(s.N, dtype=np.float32)
            b[0::s.M] = np.float32(synth.SKEW_BETA[(s.M, s.k)])
            d["b_r"] = torch.from_numpy(b).cuda()
        layer = Layer(rsq, s, d)
        steps = max(2, min(args.steps, 20))
        res = time_steps(layer, steps, 2, None, lambda: None)
        dense_ms = time_dense(rsq, s, d, steps, 1, None) / steps
        gq_ms = time_layer(rsq, s, d, steps, 1, None) / steps
        counts = layer.counts.view(s.N, s.B).sum(dim=1).cpu().numpy().reshape(s.G, s.M)
        attn_s = res["per_call_ms"]["attention"] / steps / 1e3
        ach = flops(s)["attention"] / attn_s / 1e12
        rows.append({"workload": f"{name} ({'skewed' if skew else 'balanced'}): {describe(s)}",
                     "steps": steps, "gqe_ms": gq_ms, "dense_ms": dense_ms,
                     "speedup": dense_ms / gq_ms,
                     "hot_expert_share": float(counts[:, 0].sum()) / (s.G * s.R),
                     "attn_tflops": ach, "attn_frac_of_bf16_peak": ach / pk["bf16"],
                     "breakdown_ms": {c: v / steps for c, v in res["per_call_ms"].items()},
                     "fractions": call_fractions(s, res["per_call_ms"], steps, pk)})
        if rsq.gqe_read_status() != 0:
            raise RuntimeError(f"device-side status set in pool sweep {name}")
        del layer, d
        torch.cuda.empty_cache()
    return rows


def run_reference(args):
    """The fp64 oracle on the host cores, on prefixes of the workload sized so
    that warmup + steps end within about two minutes."""
    import oracle  # noqa: F401
    shape = WORKLOADS[args.workload]
    budget = 120.0 / (args.steps + max(1, args.warmup))
    T = shape.T
    probe = cpu_baseline(shape, max_tokens=min(T, 256))
    per_tok = probe["seconds"] / min(T, 256)
    while T > 256 and per_tok * T * (1 + T / 4096) > budget:
        T //= 2
    for _ in range(max(1, args.warmup) if T <= 256 else 1):
        cpu_baseline(shape, max_tokens=T)
    times = []
    for _ in range(args.steps):
        times.append(cpu_baseline(shape, max_tokens=T)["seconds"])
    value = T * args.steps / sum(times)
    from threadpoolctl import threadpool_info
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(times) / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {describe(shape)}", "global_batch": shape.B,
                   "seq_len": shape.T, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: the full oracle layer on the first {T} of {shape.T} "
                                   f"tokens of the sequence (a causal prefix), fp64 numpy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default=HEADLINE)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--sweep-max", choices=SWEEP, default=None)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-pool", action="store_true",
                    help="skip the expert-pool workloads (32 experts, k = 1, 2; skewed, balanced)")
    ap.add_argument("--backward", action="store_true",
                    help="time only the layer backward (gqe_layer_bwd) on --workload, --steps calls")
    args = ap.parse_args()
    if args.backward:
        import routed_sparse_query_b200 as rsq
        shape = WORKLOADS[args.workload]
        d = device_inputs_from_synth(synth.make_layer_inputs(shape))
        print(json.dumps(backward_bench(rsq, shape, d, steps=args.steps)), flush=True)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    dist = None
    if world > 1:
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        out = run_ours(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
