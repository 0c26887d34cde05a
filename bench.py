"""Benchmark of the ExpertsInt8 MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl jmoe|reference]

A step is one pass of the per-token hot path -- router (logits, softmax,
top-2), grouping by expert, gate/up GEMM with in-kernel INT8->BF16
dequantisation and SwiGLU, down GEMM, gate-weighted combine -- over one batch
of synthetic tokens, with the weights (quantised once at load time, as the
method prescribes) resident in HBM.  The headline workload is the
Jamba-1.5-Mini-shaped decode batch (T = 8 tokens, d_model 4096, d_ff 14336,
16 experts, top-2); the other workloads are reported under "also".

With N > 1 (torchrun), every rank runs its own independent batch (the layer
is per-token: no data-path collective) and rank 0 prints the aggregate.

--impl reference times the CPU oracle on this machine's host cores on a
bounded sample of the same workload (the pages ship no code to run).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from synth.workloads import (LARGE_DECODE, LARGE_PREFILL_SKEW, MINI_DECODE,  # noqa: E402
                             MINI_DECODE_E64, MINI_DENSE, MINI_PREFILL, SIGMA_R, SIGMA_W, SIGMA_X,
                             TINY, Workload)

HEADLINE = MINI_DECODE
METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill TFLOPS as % of B200 roofline"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# B200 dense BF16 tensor-core rate from the data sheet (the 4.5 PFLOP/s figure
# is with 2:4 sparsity); reported beside the measured peaks, for context.
SPEC_BF16_DENSE_TFLOPS = 2250.0


# ----------------------------------------------------------------------------- clocks


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while running."""

    NAMES = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int, period_s: float = 0.002):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._halt = threading.Event()
        self.handle = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            uuid = getattr(props, "uuid", None)
            h = None
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device)
            self.handle = h
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # NVML unavailable: report it
            self.error = str(exc)

    def run(self):
        if self.handle is None:
            return
        n = self.nvml
        while not self._halt.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
                self.reasons |= int(n.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"]}
        reasons = [name for bit, name in self.NAMES.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- device layer


class Layer:
    """One MoE layer's device tensors: seeded inputs, weights quantised once."""

    def __init__(self, wl: Workload, device):
        import torch

        import int8_weight_moe_b200 as jm

        self.wl, self.device = wl, device
        s, E, d, f = wl.seed, wl.E, wl.d_model, wl.d_ff
        self.x = synth.normal_bf16_gpu(s, synth.X, SIGMA_X, (wl.T, d), device=device)
        self.w_router = None if wl.dense else synth.normal_f32_gpu(s, synth.WR, SIGMA_R, (E, d),
                                                                   device=device)
        self.bias = (torch.tensor(wl.bias, dtype=torch.float32, device=device)
                     if wl.bias is not None else None)
        w = synth.normal_bf16_gpu(s, synth.WGU, SIGMA_W, (E, 2 * f, d), device=device)
        self.w_gu, self.s_gu = jm.jmoe_quantize(w)
        del w
        w = synth.normal_bf16_gpu(s, synth.WD, SIGMA_W, (E, d, f), device=device)
        self.w_d, self.s_d = jm.jmoe_quantize(w)
        del w
        torch.cuda.synchronize(device)
        self.desc = jm.make_desc(self.w_gu, self.s_gu, self.w_d, self.s_d, top_k=wl.top_k)
        self.out = torch.empty_like(self.x)
        if wl.dense:
            self.ws = torch.empty(jm.jmoe_mlp_workspace_size(wl.T, d, f), dtype=torch.uint8,
                                  device=device)
        else:
            self.ids = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device=device)
            self.gates = torch.empty((wl.T, wl.top_k), dtype=torch.float32, device=device)
            self.ws = torch.empty(jm.jmoe_forward_workspace_size(self.desc, wl.T),
                                  dtype=torch.uint8, device=device)

    def step(self, x=None, out=None, route_events=None):
        """One pass of the hot path on the current stream."""
        import int8_weight_moe_b200 as jm

        x = self.x if x is None else x
        out = self.out if out is None else out
        if self.wl.dense:
            jm.jmoe_mlp_forward(x, self.w_gu[0], self.s_gu[0], self.w_d[0], self.s_d[0], out=out,
                                workspace=self.ws)
            return
        if route_events:
            route_events[0].record()
        jm.jmoe_route(x, self.w_router, self.wl.top_k, self.bias, topk_ids=self.ids,
                      topk_w=self.gates)
        if route_events:
            route_events[1].record()
        jm.jmoe_forward(self.desc, x, self.ids, self.gates, out=out, workspace=self.ws)

    def prefill_path(self):
        """Whether the library's automatic choice is the tensor-core path here
        (the two paths need different workspaces, which reveals the choice)."""
        import int8_weight_moe_b200 as jm

        return jm.uses_prefill_path(self.desc, self.wl.T)

    def touched_experts(self):
        if self.wl.dense:
            return 1
        return int(np.unique(self.ids.cpu().numpy()).size)

    def weight_bytes(self):
        return self.w_gu.numel() + self.w_d.numel()

    def expert_counts(self):
        """Token->expert assignments per expert in the last routing."""
        if self.wl.dense:
            return np.array([self.wl.T])
        return np.bincount(self.ids.cpu().numpy().reshape(-1), minlength=self.wl.E)


def dequant_conversions(counts, d: int, f: int, prefill: bool) -> int:
    """INT8 -> 16-bit weight conversions one step of the expert kernels makes
    (the dequantisation work, reported apart from the FLOPs).  The decode
    kernels convert an expert's 3*d*f weights once per pass over up to 8 of
    its tokens; the tensor-core kernels once per 512-row tile of its rows,
    which are padded to a multiple of 128."""
    total = 0
    for c in counts:
        c = int(c)
        if c <= 0:
            continue
        if prefill:
            padded = -(-c // 128) * 128
            passes = -(-padded // 512)
        else:
            passes = -(-c // 8)
        total += passes * 3 * d * f
    return total


def kernel_work(layer: Layer):
    """Algorithmic work of the dominant kernel (the gate/up GEMM) per launch
    and of the whole step.  HBM regime: the gate/up GEMV must read the int8
    gate/up rows of every touched expert (2*f*d bytes each) and each token's
    activation row once (2*d bytes); the step must read all three matrices of
    every touched expert, their fp32 scales, and the tokens in and out.
    Tensor-core regime: 2 FLOPs per multiply-add, 2*f*d per assignment for
    gate/up, 3*f*d for the whole step."""
    wl = layer.wl
    d, f, A, T = wl.d_model, wl.d_ff, wl.A, wl.T
    touched = layer.touched_experts()
    gu_bytes = touched * 2 * f * d + T * d * 2
    step_bytes = touched * 3 * d * f + touched * (2 * f + d) * 4 + T * d * 2 * 2
    conv = dequant_conversions(layer.expert_counts(), d, f, layer.prefill_path())
    return {"touched": touched, "gate_up_bytes": gu_bytes, "step_bytes": step_bytes,
            "gate_up_flops": 4 * A * d * f, "step_flops": 6 * A * d * f,
            "dequant": {"int8_conversions_per_step": conv,
                        "per_touched_weight": round(conv / (touched * 3 * d * f), 3)}}


def _primed_events(n: int):
    """n timing events whose CUDA handles already exist (torch creates the
    handle on the first record; the library re-records them later)."""
    import torch

    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for ev in evs:
        ev.record()
    return evs


def step_percentiles(ms_list):
    """Median, 10th and 90th percentile of per-step times (ms)."""
    xs = np.asarray(ms_list, dtype=np.float64)
    return {"median": round(float(np.median(xs)), 4), "p10": round(float(np.percentile(xs, 10)), 4),
            "p90": round(float(np.percentile(xs, 90)), 4)}


def timed_run(layer: Layer, steps: int, warmup: int, dist_on: bool,
              stages=("gate_up",), route: bool = False, spread=None):
    """Warm-up, then exactly `steps` timed steps between barriers.  Inside the
    timed region the library records a CUDA event pair on the launching
    stream around each stage named in `stages` (and the bench around the
    router if `route`); the other stages record nothing, so the step pays
    only for the events it needs.  Returns (total ms, mean ms per recorded
    stage that ran, kernel launches in the timed region); if `spread` is a
    dict, it receives the per-step percentiles of each recorded stage."""
    import torch

    import int8_weight_moe_b200 as jm

    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    want = [i for i, name in enumerate(jm.STAGES) if name in stages]
    stage_events, route_events = [], []
    for _ in range(steps):
        evs = [None] * (2 * len(jm.STAGES))
        primed = _primed_events(2 * len(want))
        for j, i in enumerate(want):
            evs[2 * i], evs[2 * i + 1] = primed[2 * j], primed[2 * j + 1]
        stage_events.append(evs)
        route_events.append(_primed_events(2) if route else None)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    n0 = jm.jmoe_launch_count()
    start.record()
    for i in range(steps):
        if want:
            jm.jmoe_profile_events(stage_events[i])
        layer.step(route_events=route_events[i])
    stop.record()
    launches = jm.jmoe_launch_count() - n0
    jm.jmoe_profile_events(None)
    torch.cuda.synchronize()
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
    total_ms = start.elapsed_time(stop)
    out = {}
    if route and not layer.wl.dense:
        out["route"] = sum(a.elapsed_time(b) for a, b in route_events) / len(route_events)
    for i in want:
        pairs = [(evs[2 * i], evs[2 * i + 1]) for evs in stage_events]
        # a stage that does not run on this path leaves its primed pair, which
        # spans no step: report only stages whose events moved
        if stage_ran(pairs, start):
            per_step = [a.elapsed_time(b) for a, b in pairs]
            out[jm.STAGES[i]] = sum(per_step) / len(per_step)
            if spread is not None:
                spread[jm.STAGES[i]] = step_percentiles(per_step)
    return total_ms, out, launches


def stage_breakdown(layer: Layer, steps: int, dist_on: bool):
    """Mean ms of every stage (and the router), from a separate pass with an
    event pair around each of them."""
    import int8_weight_moe_b200 as jm

    _, stages, _ = timed_run(layer, steps, 3, dist_on, stages=jm.STAGES, route=True)
    return stages


def stage_ran(pairs, start):
    """True when the stage's events were re-recorded after `start`."""
    try:
        return all(start.elapsed_time(a) >= 0 and a.elapsed_time(b) >= 0 for a, b in pairs)
    except RuntimeError:
        return False


def sources_sha256(paths):
    """sha256 over the listed source files (repo-relative), in order."""
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profile_traffic(workload: str, stage: str):
    """DRAM bytes per launch (read + write) of the kernel behind `stage` on
    `workload`, from an ncu summary under profiles/ (see profile_figure)."""
    v = profile_figure(workload, stage, "traffic_bytes_per_launch")
    return None if v is None else int(float(v))


def profile_figure(workload: str, stage: str, key: str):
    """A figure of the kernel behind `stage` on `workload` from an ncu summary
    under profiles/.  Each summary lists its figures as "- key: value" lines:
    stage, workload, the figures (traffic_bytes_per_launch,
    tensor_pipe_active_pct, ...), sources and sources_sha256.  None when no
    summary matches or when any of the kernel's sources changed since the
    capture (the counters then describe another kernel)."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for name in sorted(os.listdir(pdir)):
        if not name.endswith(".md"):
            continue
        kv = {}
        with open(os.path.join(pdir, name)) as fh:
            for line in fh:
                if line.startswith("- ") and ": " in line:
                    k, v = line[2:].split(": ", 1)
                    kv[k.strip()] = v.strip().strip("`")
        if kv.get("stage") != stage or kv.get("workload") != workload:
            continue
        if key not in kv or "sources" not in kv:
            continue
        try:
            if sources_sha256(kv["sources"].split()) != kv.get("sources_sha256"):
                return None
        except OSError:
            return None
        v = kv[key].split()[0]
        return float(v) if "." in v else int(v)
    return None


def roofline_entry(layer: Layer, stages: dict, peaks: dict):
    work = kernel_work(layer)
    traffic = profile_traffic(layer.wl.name, "gate_up")
    ms = stages.get("gate_up")
    if ms is None or ms <= 0:
        return None
    if layer.prefill_path():
        # The target's dense BF16 peak is the measured rate of a cuBLAS GEMM
        # timed alone (`bf16_tflops`); the power-capped sustained rate and the
        # data-sheet figure ride along.
        achieved = work["gate_up_flops"] / (ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        return {"bound": "tensor", "kernel": "gate_up", "achieved": round(achieved, 2),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": traffic, "ms": round(ms, 4),
                "peak_source": peaks["source"] + " burst bf16 (dense cuBLAS GEMM timed alone)",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "sustained_peak": peaks["bf16_tflops_sustained"],
                "frac_of_spec_dense": round(achieved / SPEC_BF16_DENSE_TFLOPS, 4),
                "tensor_pipe_active": profile_figure(layer.wl.name, "gate_up",
                                                     "tensor_pipe_active_pct")}
    achieved = work["gate_up_bytes"] / (ms * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "kernel": "gate_up", "achieved": round(achieved, 1), "peak": peak,
            "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
            "ms": round(ms, 4), "peak_source": peaks["source"] + " hbm copy"}


def graph_run(layer: Layer, steps: int, warmup: int = 3, prologue: bool = True):
    """The whole layer -- with its RMSNorm prologue (RMSNorm + router +
    experts) or without it (router + experts, the timed eager step's work) --
    captured once in a CUDA graph (int8_weight_moe_b200.MoeLayerGraph) and
    replayed; ms per replay from CUDA events on the replay stream."""
    import torch

    import int8_weight_moe_b200 as jm

    wl = layer.wl
    gamma = None
    if prologue:
        gamma = (synth.normal_bf16_gpu(wl.seed + 7, synth.X, 0.25, (wl.d_model,),
                                       device=layer.device).float() + 1.0).to(torch.bfloat16)
    g = jm.MoeLayerGraph(layer.desc, layer.w_router, wl.T, gamma=gamma, eps=1e-6,
                         bias=layer.bias)
    g.x.copy_(layer.x)
    for _ in range(warmup):
        g.run()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        g.run()
    stop.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop) / steps
    what = " + RMSNorm prologue" if prologue else " (router + experts, as the eager step)"
    return {"workload": wl.name + what + ", CUDA graph", "ms_per_step": round(ms, 4),
            "tokens_per_s": round(wl.T / (ms * 1e-3), 1)}


def e2e_run(layer: Layer, steps: int, warmup: int, dist_on: bool = False):
    """Same metric through the public API with host buffers: per step a
    host->device copy of the tokens from pinned memory and a device->host read
    of the layer output, inside the timed region.  As a serving loop would run
    it: the copies go on a second stream into double buffers, so step i+1's
    tokens come in and step i's output goes out while the next step computes
    (the copies of a step never overlap that step's own kernels).  `serial`
    is the same with every copy on the compute stream between the steps."""
    import torch

    wl = layer.wl
    xh = layer.x.cpu().pin_memory()
    oh = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    xd = [torch.empty_like(layer.x) for _ in range(2)]
    od = [torch.empty_like(layer.out) for _ in range(2)]
    comp = torch.cuda.current_stream()
    copy = torch.cuda.Stream()

    def serial(n):
        for _ in range(n):
            xd[0].copy_(xh, non_blocking=True)
            layer.step(x=xd[0], out=od[0])
            oh.copy_(od[0], non_blocking=True)

    def pipelined(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        copy.wait_stream(comp)
        with torch.cuda.stream(copy):
            xd[0].copy_(xh, non_blocking=True)
            ev_in[0].record()
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                with torch.cuda.stream(copy):
                    if i >= 1:
                        copy.wait_event(ev_done[1 - b])  # step i - 1 no longer reads its buffer
                    xd[1 - b].copy_(xh, non_blocking=True)
                    ev_in[1 - b].record()
            comp.wait_event(ev_in[b])
            if i >= 2:
                comp.wait_event(ev_out[b])  # step i - 2's output has left od[b]
            layer.step(x=xd[b], out=od[b])
            ev_done[b].record()
            with torch.cuda.stream(copy):
                copy.wait_event(ev_done[b])
                oh.copy_(od[b], non_blocking=True)
                ev_out[b].record()
        comp.wait_stream(copy)

    out = {}
    for name, fn in (("pipelined", pipelined), ("serial", serial)):
        fn(warmup)
        torch.cuda.synchronize()
        if dist_on:
            import torch.distributed as dist

            dist.barrier()
            torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        start.record()
        fn(steps)
        stop.record()
        torch.cuda.synchronize()
        out[name] = start.elapsed_time(stop) / steps
    ms = out["pipelined"]
    nbytes = wl.T * wl.d_model * 2
    return {"value": round(wl.T / (ms * 1e-3), 1), "unit": UNIT, "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
            "copies": "double-buffered on a second stream, overlapping the neighbouring steps",
            "serial": {"ms_per_step": round(out["serial"], 4),
                       "value": round(wl.T / (out["serial"] * 1e-3), 1)}}


# ----------------------------------------------------------------------------- CPU oracle


def oracle_threads():
    if os.environ.get("OMP_NUM_THREADS"):
        return int(os.environ["OMP_NUM_THREADS"])
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


class OracleRun:
    """The CPU oracle on a sample of a workload's tokens (weights generated
    and quantised on the host for the experts the sample touches)."""

    def __init__(self, wl: Workload, tokens):
        import oracle

        self.o = oracle
        self.wl = wl
        s, E, d, f = wl.seed, wl.E, wl.d_model, wl.d_ff
        self.tokens = np.asarray(tokens)
        self.x = synth.normal_bf16_bits(s, synth.X, SIGMA_X, (wl.T, d))[self.tokens]
        self.wr = None if wl.dense else synth.normal_f32(s, synth.WR, SIGMA_R, (E, d))
        self.bias = None if wl.bias is None else np.array(wl.bias, dtype=np.float32)
        if wl.dense:
            ids = np.zeros((len(self.tokens), 1), dtype=np.int32)
        else:
            _, ids, _ = oracle.route(self.x, self.wr, wl.top_k, self.bias)
        self.tables = [[None] * E for _ in range(4)]
        for e in sorted(set(int(v) for v in ids.reshape(-1))):
            wgu = synth.normal_bf16_bits(s, synth.WGU, SIGMA_W, (2 * f, d), start=e * 2 * f * d)
            qg, sg = oracle.quantize(wgu)
            del wgu
            wdn = synth.normal_bf16_bits(s, synth.WD, SIGMA_W, (d, f), start=e * d * f)
            qd, sd = oracle.quantize(wdn)
            del wdn
            for i, a in enumerate((qg, sg, qd, sd)):
                self.tables[i][e] = a

    def step(self):
        """Route, group and run the experts for the sample; returns #tokens."""
        if self.wl.dense:
            e = 0
            self.o.mlp_forward(self.x, self.tables[0][e], self.tables[1][e], self.tables[2][e],
                               self.tables[3][e])
        else:
            _, ids, g = self.o.route(self.x, self.wr, self.wl.top_k, self.bias)
            self.o.permute(ids, self.wl.E)
            self.o.moe_forward(self.x, ids, g, *self.tables)
        return len(self.tokens)


# Tokens of the CPU-baseline sample: a whole decode-sized batch, else a slice
# (the oracle's cost per token is the same for every token: its weights stay
# INT8 + scale and each assignment streams one expert's matrices).
CPU_SAMPLE_MAX_TOKENS = 64
CPU_SAMPLE_SLICE = 256


def cpu_sample_tokens(wl: Workload) -> np.ndarray:
    if wl.T <= CPU_SAMPLE_MAX_TOKENS:
        return np.arange(wl.T)
    # a seeded slice spread over the batch
    rng = np.random.default_rng(wl.seed)
    return np.sort(rng.choice(wl.T, size=CPU_SAMPLE_SLICE, replace=False))


def cpu_baseline(wl: Workload, budget_s: float = 8.0, max_reps: int = 50):
    """The oracle on the host cores: route + group + experts over the sample,
    repeated until `budget_s` has passed; tokens/s over the sample."""
    tokens = cpu_sample_tokens(wl)
    run = OracleRun(wl, tokens)
    t0 = time.perf_counter()
    n = 0
    reps = 0
    while True:
        n += run.step()
        reps += 1
        if time.perf_counter() - t0 >= budget_s or reps >= max_reps:
            break
    dt = time.perf_counter() - t0
    what = ("all" if len(tokens) == wl.T else "a seeded slice of") + f" {len(tokens)} tokens"
    return {"value": round(n / dt, 3), "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{wl.name}: {what} x {reps} repetitions (route + group + experts, "
                      f"fp64 C oracle), {dt:.1f} s; tokens/s of the sample stands for the "
                      "batch (per-token cost is the same for every token)"}


def reference_arm(args):
    """--impl reference: the oracle on the host cores, on the headline config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = HEADLINE
    run = OracleRun(wl, np.arange(1))  # one token (two expert assignments) per step
    for _ in range(args.warmup):
        run.step()
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += run.step()
    dt = time.perf_counter() - t0
    value = n / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**wl.describe(), "sample_tokens_per_step": 1},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle_threads(),
                             "kind": "oracle",
                             "sample": f"{wl.name}: 1 token per step (route + group + 2 experts)"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- ranks


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (every rank gets it); the value
    itself without a process group.  Timings are combined this way: the job
    takes as long as its slowest rank."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Weak scaling: every rank processes its own batch of `tokens_per_rank`
    tokens per step, so the job processes world * tokens_per_rank per step."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="jmoe", choices=["jmoe", "reference"])
    ap.add_argument("--no-also", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--only", default=None, help="run only this workload (name) as headline")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the token count of --only (profiling runs on smaller cases)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        reference_arm(args)
        return

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import int8_weight_moe_b200 as jm

    peaks = load_peaks()
    wl = HEADLINE
    if args.only:
        from synth.workloads import BY_NAME

        wl = BY_NAME[args.only]
        if args.tokens:
            import dataclasses

            wl = dataclasses.replace(wl, T=args.tokens, name=f"{wl.name}@T{args.tokens}")
    layer = Layer(wl, torch.device("cuda", local))

    sampler = ClockSampler(local)
    sampler.start()
    # The headline pass records no events: an event between two kernels
    # chained by programmatic dependent launch makes the second wait for the
    # first to finish, which costs the step its launch overlap (measured: 5%
    # of a Mini decode step).  The dominant kernel's duration comes from a
    # second timed pass of the same length with an event pair around it.
    total_ms, _, launches = timed_run(layer, args.steps, args.warmup, dist_on, stages=())
    clocks = sampler.stop()
    spread = {}
    _, stages, _ = timed_run(layer, args.steps, 3, dist_on, spread=spread)
    dev = torch.device("cuda", local)
    total_ms = max_over_ranks(total_ms, dev)
    ms = total_ms / args.steps
    value = whole_job_tokens_per_s(world, wl.T, ms)
    roof = roofline_entry(layer, stages, peaks)
    if roof is not None and "gate_up" in spread:
        # the dominant kernel's per-launch spread over the timed steps
        roof["ms_per_launch"] = spread["gate_up"]
    breakdown = stage_breakdown(layer, min(args.steps, 50), dist_on)
    e2e = e2e_run(layer, max(args.steps // 2, 10), 3, dist_on)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], dev)
    e2e["ms_per_step"] = round(e2e_ms, 4)
    e2e["value"] = round(whole_job_tokens_per_s(world, wl.T, e2e_ms), 1)
    graph_line = None
    if not wl.dense:
        graph_line = graph_run(layer, max(args.steps // 2, 10))
        # like for like with the timed eager step: the same kernels, replayed
        graph_line["without_prologue"] = graph_run(layer, max(args.steps // 2, 10),
                                                   prologue=False)
    work = kernel_work(layer)
    step_gbs = work["step_bytes"] / (ms * 1e-3) / 1e9
    del layer
    torch.cuda.empty_cache()

    also = []
    if not args.no_also and not args.only:
        for other in (TINY, MINI_PREFILL, MINI_DENSE, LARGE_DECODE, LARGE_PREFILL_SKEW,
                      MINI_DECODE_E64):
            lay = Layer(other, torch.device("cuda", local))
            steps = 20 if other.regime == "prefill" else 100
            tms, _, _ = timed_run(lay, steps, 3, dist_on, stages=())
            _, st, _ = timed_run(lay, steps, 3, dist_on)
            oms = max_over_ranks(tms, dev) / steps
            bd = stage_breakdown(lay, steps, dist_on)
            w2 = kernel_work(lay)
            entry = {"workload": other.name, "tokens_per_s": round(whole_job_tokens_per_s(world, other.T, oms), 1),
                     "ms_per_step": round(oms, 4), "path": "prefill" if lay.prefill_path() else "decode",
                     "stages_ms": {k: round(v, 4) for k, v in bd.items()},
                     "roofline": roofline_entry(lay, st, peaks),
                     "step_hbm_gbs": round(w2["step_bytes"] / (oms * 1e-3) / 1e9, 1),
                     "step_tflops": round(w2["step_flops"] / (oms * 1e-3) / 1e12, 2),
                     "dequant": w2["dequant"]}
            del lay
            torch.cuda.empty_cache()
            if rank == 0 and world == 1 and not args.no_cpu:
                entry["cpu_baseline"] = cpu_baseline(other)
            also.append(entry)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {**wl.describe(),
                           "weights": "int8 per-output-channel (quantised once on device)",
                           "l2": "inputs larger than L2 (touched int8 weights "
                                 f"{work['touched'] * 3 * wl.d_model * wl.d_ff / 1e9:.2f} GB "
                                 "> 126 MB L2), no flush",
                           "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clocks,
                "stages_ms": {k: round(v, 4) for k, v in breakdown.items()},
                "stages_ms_source": "separate pass after the timed one, with an event pair "
                                    "around every stage",
                "roofline_source": "a second timed pass of the same steps with an event pair "
                                   "around the gate/up kernel (the headline pass records no "
                                   "events: they would cost the step its launch overlap)",
                "step_hbm_gbs": round(step_gbs, 1),
                "touched_experts": work["touched"], "dequant": work["dequant"],
                "graph": graph_line, "also": also}
        print(json.dumps(line), flush=True)
    if dist_on:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
