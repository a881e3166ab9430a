#!/usr/bin/env python
"""Benchmark of the sparse-MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one whole layer forward (router, dispatch, gate_up GEMM + SwiGLU, down GEMM with the
router weight, combine) over one batch of synthetic tokens, inputs resident in HBM.  The timed
steps replay a CUDA graph of the C-ABI call ``moe_layer_forward_timed`` (events around every
stage, recorded on the launching stream).  ``e2e`` repeats the measurement through
``moe_layer_forward_host`` with pinned host buffers (x in, y out, copies inside the timed region).
With N > 1 (torchrun) every rank runs an independent replica (weak scaling); the only
collectives are the barrier and the max-over-ranks of the elapsed time.
``--impl reference`` times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "MoE layer tokens/s at 1 B200; prefill TFLOP/s and decode active-weight GB/s vs peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (read + write) of the dominant kernel (the gate_up launch) per launch, from one ncu
# capture of the same bench command (the kernel summaries under profiles/): valid only while that
# kernel's sources are unchanged, else reported as null.
_CSRC = "sparse_mixture_experts_16_b200/csrc/"
_TRAFFIC = {
    # kernel variant -> (its sources, their sha256, {workload: dram__bytes_read.sum + dram__bytes_write.sum})
    "bf16": ((_CSRC + "grouped_gemm_sm100.cu", _CSRC + "sm100_ptx.cuh", _CSRC + "moe_common.cuh"),
             "499dcc3232d606bb964c25506e639710b704dc2792467aa0d428d086454b0888",
             {"deepseek": 16.357346e9 + 0.267214e9, "mixtral": 1.946551e9 + 0.226511e9,
              "gptoss": 1.250823e9 + 0.179702e9, "gptoss_decode_T1": 0.135693e9 + 0.003212e9,
              "gptoss_decode_T8": 0.707973e9 + 0.003855e9, "gptoss_decode_T32": 1.076509e9 + 0.003957e9,
              "gptoss_decode_T64": 1.077995e9 + 0.004742e9, "deepseek_decode": 5.876478e9 + 0.004464e9}),
    "bf16_wide": ((_CSRC + "grouped_gemm_wide_sm100.cu", _CSRC + "sm100_ptx.cuh", _CSRC + "moe_common.cuh"),
                  "", {}),
    "bf16_pair": ((_CSRC + "grouped_gemm_pair_sm100.cu", _CSRC + "sm100_ptx.cuh", _CSRC + "moe_common.cuh"),
                  "", {}),
    "fp8": ((_CSRC + "stream_fp8w_sm100.cu", _CSRC + "sm100_ptx.cuh", _CSRC + "moe_common.cuh"),
            "bc15fd3599b4d7d25cc3852951449f0a47e6a1ae2b5adb086609c2d1f4a02174",
            {"deepseek_decode": 2.942161e9 + 0.004544e9, "gptoss_decode_T1": 0.067342e9 + 0.000812e9,
             "gptoss_decode_T8": 0.364131e9 + 0.004026e9, "gptoss_decode_T64": 0.556408e9 + 0.004305e9}),
}


def measured_traffic(workload: str, weights: str = "bf16"):
    import hashlib

    files, digest, table = _TRAFFIC[weights]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest() != digest:
        return None
    return table.get(workload)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------------- accounting
def gateup_flops(w: mi.Workload) -> float:
    """Algorithmic FLOPs of the gate_up launch: 2*D*2F per routed row, 2*D*2Fs per token."""
    return float(w.T) * (w.k * 4.0 * w.D * w.F + 4.0 * w.D * w.Fs)


def down_flops(w: mi.Workload) -> float:
    return float(w.T) * (w.k * 2.0 * w.D * w.F + 2.0 * w.D * w.Fs)


def active_weight_bytes(w: mi.Workload, n_active: int, part: str = "all", weights: str = "bf16") -> float:
    """Bytes of weights that must be streamed: distinct active experts (+ shared expert).  bf16: 2
    bytes per weight; fp8: 1 byte per E4M3 code plus a 4-byte scale per weight row."""
    if weights == "fp8":
        gu = (2.0 * w.F * w.D + 4 * 2.0 * w.F) * n_active + (2.0 * w.Fs * w.D + 4 * 2.0 * w.Fs)
        dn = (1.0 * w.D * w.F + 4.0 * w.D) * n_active + ((1.0 * w.D * w.Fs + 4.0 * w.D) if w.Fs else 0.0)
    else:
        gu = 2.0 * w.F * w.D * 2 * n_active + 2.0 * w.Fs * w.D * 2
        dn = 1.0 * w.D * w.F * 2 * n_active + 1.0 * w.D * w.Fs * 2
    return {"gate_up": gu, "down": dn, "all": gu + dn}[part]


def decode_tokens_per_s_bound(bandwidth_bytes_per_s: float, active_params: float, bytes_per_param: float) -> float:
    """The pages' decode model: tokens/s = memory bandwidth / bytes of active parameters per token
    (keryc.com, "Por que MoEs importan": gpt-oss-20b, ~3.6e9 active params, bf16, ~800 GB/s)."""
    return bandwidth_bytes_per_s / (active_params * bytes_per_param)


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", self.gpu_id, "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), sm_max=float(f[2]), power=float(f[3]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r["power"] > 300] or rows
        capped = sum(1 for r in loaded if r["pcap"] == "Active")
        reasons = set()
        for r in loaded:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["sm_max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
                "samples_power_capped": capped, "power_w_max": max(r["power"] for r in rows)}


def max_over_ranks(vals, dev, world: int):
    """Each value's maximum over the ranks, from one all-reduce (every rank calls this at the same
    point, with the same number of values).  One rank: the values unchanged."""
    vals = [float(v) for v in vals]
    if world <= 1:
        return vals
    import torch
    import torch.distributed as dist

    t = torch.tensor(vals, device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Tokens per second of the whole job: every rank ran `steps` steps of `tokens_per_step`
    tokens, and the job took as long as its slowest rank (`max_ms`, summed over the steps)."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


def tensor_peak(pk: dict, clocks: dict, timed_s: float):
    """The bf16 peak that matches the clocks of the timed region: the sustained figure (a
    seconds-long loop at the 1 kW power cap) only for a region of >= 1 s in which the sampler saw
    sw_power_cap under load; otherwise the burst figure (a GEMM timed alone at full clocks).
    Returns (peak TFLOP/s, which)."""
    if timed_s >= 1.0 and clocks.get("samples_power_capped", 0) > 0:
        return pk["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return pk["bf16_tflops"], "bf16_tflops"


# ---------------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """The fp64 oracle, as it stands, on a bounded sample of the workload's tokens (all host
    cores; with fp8 weights the oracle's E4M3 layer on weights it quantised itself).  Preparing the
    sample (routing a prefix of the tokens, generating the weights of the experts the sample
    needs, at most ``weight_budget`` bytes of them) happens once, outside any timed call."""

    def __init__(self, w: mi.Workload, weights: str = "bf16", weight_budget: float = 3.0e9):
        import oracle

        self.w, self.weights, self.cores = w, weights, host_cores()
        wg = mi.host_wg(w)
        bias = mi.bias_f32(w)
        expert_bytes = 3.0 * w.D * w.F * 2
        max_experts = max(w.k, min(40, int(weight_budget // expert_bytes)))
        # route a prefix of tokens to know which experts the sample needs
        probe = np.arange(min(w.T, 256))
        xp = mi.host_x(w, rows=probe)
        idx, _ = oracle.router(xp, wg, bias, w.k)
        chosen, experts = [], set()
        for i in range(len(probe)):
            e = set(idx[i].tolist())
            if len(experts | e) > max_experts and chosen:
                continue
            experts |= e
            chosen.append(i)
        experts = sorted(experts)
        gu = dict(zip(experts, mi.host_gate_up(w, experts)))
        dn = dict(zip(experts, mi.host_down(w, experts)))
        sgu, sdn = mi.host_shared(w)
        if weights == "fp8":
            q = dict(gu_q={}, gu_s={}, dn_q={}, dn_s={})
            for e in experts:
                q["gu_q"][e], q["gu_s"][e] = oracle.quantize_rows_fp8(gu[e])
                q["dn_q"][e], q["dn_s"][e] = oracle.quantize_rows_fp8(dn[e])
            shared_q = None
            if w.Fs:
                a, b = oracle.quantize_rows_fp8(sgu)
                c, d = oracle.quantize_rows_fp8(sdn)
                shared_q = dict(gu_q=a, gu_s=b, dn_q=c, dn_s=d)
            self.run = lambda x: oracle.layer_fp8(x, wg, bias, w.k, q, shared_q)  # noqa: E731
        else:
            self.run = lambda x: oracle.layer(x, wg, bias, gu, dn, w.k, sgu, sdn, nthreads=self.cores)  # noqa: E731
        self.x = xp[np.array(chosen)]
        self.n_distinct = len(chosen)

    def rate(self, budget_s: float = 12.0):
        """Time growing batches of sampled tokens until about ``budget_s`` of oracle time has passed.
        Returns (tokens/s, tokens timed, seconds)."""
        n, done, elapsed = min(len(self.x), self.cores), 0, 0.0
        while True:
            x = self.x[np.arange(done, done + n) % len(self.x)]
            t0 = time.perf_counter()
            self.run(x)
            dt = time.perf_counter() - t0
            done += n
            elapsed += dt
            if elapsed >= budget_s or done >= 64 * self.cores:
                break
            n = max(1, int(n * min(4.0, max(1.5, (budget_s - elapsed) / max(dt, 1e-3)))))
        return done / elapsed, done, elapsed

    def describe(self, done: int, elapsed: float) -> str:
        w = self.w
        return (f"{done} tokens of workload {w.name} (drawn from {self.n_distinct} distinct tokens; full layer: "
                f"routing over all E experts, top-{w.k} SwiGLU experts{', shared expert' if w.Fs else ''}"
                f"{', E4M3 weights' if self.weights == 'fp8' else ''}) through the fp64 oracle on {self.cores} "
                f"threads; tokens/s = {done} / {elapsed:.2f} s")


def cpu_oracle_rate(w: mi.Workload, budget_s: float = 12.0, weights: str = "bf16"):
    """(tokens/s, cores, description) of the oracle on a bounded sample of the workload."""
    sample = OracleSample(w, weights)
    v, done, elapsed = sample.rate(budget_s)
    return v, sample.cores, sample.describe(done, elapsed)


# ---------------------------------------------------------------------------------- GPU arm
def tiling_flag(tiling: str) -> int:
    import sparse_mixture_experts_16_b200 as moe

    return {"auto": 0, "row": moe.MOE_FLAG_PREFILL_ROW_TILES, "wide": moe.MOE_FLAG_PREFILL_WIDE_TILES,
            "pair": moe.MOE_FLAG_PREFILL_PAIR_TILES}[tiling]


def run_ours(args, w: mi.Workload, rank: int, world: int, local_rank: int):
    import ctypes

    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_16_b200 as moe

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    pk, pk_kind = peaks()
    with torch.cuda.stream(stream):
        inp = mi.device_inputs(w, device=dev)
        if args.weights == "fp8":
            # per-row E4M3 codes + fp32 scales, made on the device before timing; the bf16 copies go
            scales = {}
            for name in ("gate_up", "down", "shared_gate_up", "shared_down"):
                if inp[name] is not None:
                    inp[name], scales[name] = moe.moe_quantize_rows_fp8(inp[name], stream=stream)
            stream.synchronize()
            torch.cuda.empty_cache()
        else:
            scales = None
        layer = moe.MoELayer(inp["wg"], inp["gate_up"], inp["down"], w.k, bias=inp["bias"],
                             shared_gate_up=inp["shared_gate_up"], shared_down=inp["shared_down"], scales=scales,
                             flags=0 if scales is not None else tiling_flag(args.tiling))
        x = inp["x"]
        y = torch.empty_like(x)
        ws = layer.workspace(w.T)
        n_kernels = layer.kernel_count(w.T)
        weight_bytes = sum(t.numel() * t.element_size() for t in (inp["gate_up"], inp["down"], inp["wg"]))
        # a decode step touches only its active experts (as little as ~L2's size at T = 1), so decode
        # steps always start from a flushed L2; prefill steps stream weights far larger than L2
        flush = (torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
                 if weight_bytes < 8 * L2_BYTES or w.T <= 64 else None)
        flush_sum = torch.empty((), dtype=torch.int64, device=dev)

        def flush_l2(v):
            # write a buffer of twice L2's size, then read it back: L2 ends up holding only clean
            # lines of this buffer, so the timed step neither hits in L2 nor pays for writing back
            # the flush's dirty lines
            flush.fill_(v)
            torch.sum(flush, dim=0, dtype=torch.int64, out=flush_sum)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for e in evs:
            e.record(stream)
        for _ in range(max(args.warmup, 3)):
            layer.forward(x, y, stream=stream)
        stream.synchronize()
        if layer.device_error(stream) != 0:
            raise RuntimeError("device error during warm-up")
        # the timed step: a CUDA graph of moe_layer_forward_timed (stage events inside the graph)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            layer.forward_timed(x, y, evs, stream=stream)
        # the same step without stage events: the step time the bench reports
        graph_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_plain, stream=stream):
            layer.forward(x, y, stream=stream)
        for _ in range(3):
            graph.replay()
            graph_plain.replay()
        stream.synchronize()
        # active experts (for the decode byte count)
        idx, _ = moe.moe_router_topk(x, inp["wg"], inp["bias"], w.k, stream=stream)
        n_active = int(torch.unique(idx).numel())
        stream.synchronize()

    gpu_id = str(local_rank)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass

    step_ms, stage_ms = [], [[] for _ in range(5)]
    plain_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk, torch.cuda.stream(stream):
        t_begin = time.perf_counter()
        # (1) the step as the bench reports it: back-to-back graph replays, events around each
        for s in range(args.steps):
            if flush is not None:
                flush_l2(s)  # evict the weights from L2 (outside the step's events)
            plain_ev[s][0].record(stream)
            graph_plain.replay()
            plain_ev[s][1].record(stream)
        stream.synchronize()
        plain_ms = [a.elapsed_time(b) for a, b in plain_ev]
        # (2) the same step with stage events inside the graph (per-kernel roofline)
        for s in range(args.steps):
            if flush is not None:
                flush_l2(s)  # evict the weights from L2 (outside the stage events)
            graph.replay()
            stream.synchronize()
            step_ms.append(evs[0].elapsed_time(evs[5]))
            for j in range(5):
                stage_ms[j].append(evs[j].elapsed_time(evs[j + 1]))
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t_begin
    staged_ms_per_step = sum(step_ms) / len(step_ms)
    (total_ms,) = max_over_ranks([sum(plain_ms)], dev, world)
    if world > 1:
        dist.barrier()
    ms_per_step = total_ms / len(plain_ms)
    value = whole_job_rate(world, w.T, len(plain_ms), total_ms)

    # ---- end to end through the public API with pinned host buffers
    x_h = x.cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            layer.forward_host(x_h, y_h, stream=stream)
        stream.synchronize()
        e2e_steps = max(5, min(args.steps, 50))
        e2e_ms = 0.0
        for _ in range(e2e_steps):  # one step at a time: copy in, forward, copy out, synchronise
            if flush is not None:
                flush_l2(1)
            e0.record(stream)
            layer.forward_host(x_h, y_h, stream=stream)
            e1.record(stream)
            stream.synchronize()
            e2e_ms += e0.elapsed_time(e1)
    e2e_pipe_ms = None
    if flush is None:
        # Double-buffered: consecutive steps alternate between two streams, each with its own
        # workspace and pinned output buffer, so one step's host copies overlap another's compute.
        # Every step still copies its x in and its y out inside the timed region.
        s_b = torch.cuda.Stream(device=dev)
        streams = (stream, s_b)
        wss = (layer.workspace(w.T), layer.new_workspace(w.T))
        y_hs = (y_h, torch.empty_like(x_h).pin_memory())
        for i in range(4):
            layer.forward_host(x_h, y_hs[i % 2], stream=streams[i % 2], ws=wss[i % 2])
        torch.cuda.synchronize(dev)
        e0.record(stream)
        s_b.wait_event(e0)
        for i in range(e2e_steps):
            layer.forward_host(x_h, y_hs[i % 2], stream=streams[i % 2], ws=wss[i % 2])
        eb = torch.cuda.Event()
        eb.record(s_b)
        stream.wait_event(eb)
        e1.record(stream)
        stream.synchronize()
        e2e_pipe_ms = e0.elapsed_time(e1)
        del wss, y_hs
    e2e_ms, pipe_max = max_over_ranks([e2e_ms, e2e_pipe_ms or 0.0], dev, world)
    e2e_pipe_ms = pipe_max if e2e_pipe_ms is not None else None
    e2e_serial_value = whole_job_rate(world, w.T, e2e_steps, e2e_ms)
    e2e_value = whole_job_rate(world, w.T, e2e_steps, e2e_pipe_ms) if e2e_pipe_ms else e2e_serial_value

    # ---- roofline of the dominant kernel (gate_up grouped GEMM: ~2/3 of the FLOPs / weight bytes)
    clocks = clk.summary()
    gate_ms = statistics.mean(stage_ms[2])
    down_ms = statistics.mean(stage_ms[3])
    decode = w.T <= 64
    if decode:
        bytes_gu = (active_weight_bytes(w, n_active, "gate_up", args.weights) + w.T * w.k * w.D * 2.0
                    + w.T * (w.k * w.F + w.Fs) * 2.0)
        achieved = bytes_gu / (gate_ms / 1e3) / 1e9
        peak = pk["hbm_gbs"]
        fp8 = args.weights == "fp8"
        roof = {"kernel": "stream_fp8w_kernel<gate_up>" if fp8 else "grouped_gemm_kernel<gate_up, stream>",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": measured_traffic(w.name, args.weights),
                "peak_source": f"{pk_kind} hbm_gbs (copy bandwidth)"}
    else:
        achieved = gateup_flops(w) / (gate_ms / 1e3) / 1e12
        peak, which = tensor_peak(pk, clocks, wall)
        gu_kernel = {"wide_tiles": "grouped_gemm_wide_kernel<gate_up>", "pair_tiles": "grouped_gemm_pair_kernel<gate_up>"}
        path = layer.gemm_path(w.T)
        roof = {"kernel": gu_kernel.get(path, "grouped_gemm_kernel<gate_up, tiled>"),
                "bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": measured_traffic(w.name, {"wide_tiles": "bf16_wide", "pair_tiles": "bf16_pair"}.get(path, "bf16")),
                "peak_source": (f"{pk_kind} {which}: the sustained figure only for a timed region of >= 1 s "
                                f"with power-capped samples (this one: {wall:.2f} s, "
                                f"{clocks.get('samples_power_capped', 0)} capped samples)"),
                "frac_of_burst_peak": round(achieved / pk["bf16_tflops"], 4),
                "frac_of_sustained_peak": round(achieved / pk["bf16_tflops_sustained"], 4)}
    layer_tflops = w.flops / (ms_per_step / 1e3) / 1e12 * world
    layer_gbs = active_weight_bytes(w, n_active, "all", args.weights) / (ms_per_step / 1e3) / 1e9

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": len(plain_ms),
        "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "ms_per_step_with_stage_events": round(staged_ms_per_step, 4),
        "scaling": "weak", "vs_baseline": None, "dtype": "f16" if args.weights == "fp8" else "bf16",
        "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": w.name, "T": w.T, "D": w.D, "E": w.E, "k": w.k, "F": w.F, "Fs": w.Fs, "bias": w.bias,
                   "weights": ("E4M3 codes + per-row fp32 scales (f16 MMA, fp32 accumulation)"
                               if args.weights == "fp8" else "bf16"),
                   "gemm_path": layer.gemm_path(w.T),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": ("L2 flushed before every timed step (256 MB written, then read back: L2 holds clean "
                          "unrelated lines)" if flush is not None
                          else f"inputs larger than L2 (weights {weight_bytes / 1e9:.2f} GB), no flush"),
                   "timing": ("CUDA-graph replays of moe_layer_forward, events around each replay on the "
                              "launching stream; stage times from a second graph of moe_layer_forward_timed "
                              "(events between the stages), replayed in the same timed region")},
        "roofline": roof,
        "layer": {"tflops": round(layer_tflops, 1), "active_experts": n_active,
                  "active_weight_gbs": round(layer_gbs, 1),
                  "frac_tensor": round(layer_tflops / world / tensor_peak(pk, clocks, wall)[0], 4),
                  "frac_tensor_burst": round(layer_tflops / world / pk["bf16_tflops"], 4),
                  "frac_tensor_sustained": round(layer_tflops / world / pk["bf16_tflops_sustained"], 4),
                  "frac_hbm": round(layer_gbs / pk["hbm_gbs"], 4)},
        "stages_ms": {n: round(statistics.mean(v), 4) for n, v in
                      zip(("router", "dispatch", "gate_up_gemm", "down_gemm", "combine"), stage_ms)},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": w.T * w.D * 2,
                "d2h_bytes_per_step": w.T * w.D * 2,
                "api": ("moe_layer_forward_host (pinned host x, y), double-buffered: steps alternate between two "
                        "streams and two workspaces, so one step's copies overlap another's compute"
                        if e2e_pipe_ms else "moe_layer_forward_host (pinned host x, y), one step at a time"),
                "serial_value": round(e2e_serial_value, 1)},
        "gpu_launches": n_kernels * (len(plain_ms) + len(step_ms)),
        "clocks": clocks,
        "wall_s_timed_region": round(wall, 3),
    }
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            v, cores, desc = cpu_oracle_rate(w, weights=args.weights)
            result["cpu_baseline"] = {"value": round(v, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                      "sample": desc}
        print(json.dumps(result), flush=True)
    del graph, graph_plain


def run_train(args, w: mi.Workload, rank: int, world: int, local_rank: int):
    """A training step: the forward that saves the backward's inputs, then moe_layer_backward (dx and
    the fp32 weight gradients), each a CUDA graph, replayed back to back with events between them."""
    import torch

    import sparse_mixture_experts_16_b200 as moe

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    pk, pk_kind = peaks()
    with torch.cuda.stream(stream):
        inp = mi.device_inputs(w, device=dev)
        layer = moe.MoELayer(inp["wg"], inp["gate_up"], inp["down"], w.k, bias=inp["bias"],
                             shared_gate_up=inp["shared_gate_up"], shared_down=inp["shared_down"],
                             flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD | tiling_flag(args.tiling))
        x = inp["x"]
        y = torch.empty_like(x)
        dy = torch.empty_like(x)
        mi.device_fill_rows_bf16(dy, mi.STREAM_X, 1.0, seed=w.seed + 1000)
        for _ in range(max(args.warmup, 3)):
            layer.forward(x, y, stream=stream)
            dx, grads = layer.backward(x, dy, stream=stream)
        stream.synchronize()
        if layer.device_error(stream) != 0 or layer.backward_error(stream) != 0:
            raise RuntimeError("device error during warm-up")
        g_fwd, g_bwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_fwd, stream=stream):
            layer.forward(x, y, stream=stream)
        with torch.cuda.graph(g_bwd, stream=stream):
            layer.backward(x, dy, stream=stream)  # same output tensors: the layer keeps its workspaces
        for _ in range(3):
            g_fwd.replay()
            g_bwd.replay()
        stream.synchronize()
    gpu_id = str(local_rank)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_id) as clk, torch.cuda.stream(stream):
        t_begin = time.perf_counter()
        for s in range(args.steps):
            evs[s][0].record(stream)
            g_fwd.replay()
            evs[s][1].record(stream)
            g_bwd.replay()
            evs[s][2].record(stream)
        stream.synchronize()
        wall = time.perf_counter() - t_begin
    clocks = clk.summary()
    f_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in evs)
    b_ms = statistics.mean(b.elapsed_time(c) for _, b, c in evs)
    f_ms, b_ms = max_over_ranks([f_ms, b_ms], dev, world)  # the slowest rank's forward and backward
    step_ms = f_ms + b_ms
    gemm_fwd = w.T * (6.0 * w.k * w.D * w.F + 6.0 * w.D * w.Fs)
    bwd_tflops = 2 * gemm_fwd / (b_ms / 1e3) / 1e12
    peak, which = tensor_peak(pk, clocks, wall)
    n_fwd = layer.kernel_count(w.T)
    n_bwd = 9  # pad offsets, dy gather, 4 grouped GEMMs, router backward, dW_g, un-permute
    result = {
        "metric": "MoE layer training step (forward saving g|u + backward) tokens/s at 1 B200",
        "value": round(world * w.T / (step_ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": round(step_ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": w.name, "T": w.T, "D": w.D, "E": w.E, "k": w.k, "F": w.F, "Fs": w.Fs, "bias": w.bias,
                   "mode": "train", "gemm_path": layer.gemm_path(w.T), "parallelism": "single GPU",
                   "l2": f"weights {sum(t.numel() * 2 for t in (inp['gate_up'], inp['down'])) / 1e9:.2f} GB, "
                         "larger than L2, no flush",
                   "timing": "two CUDA graphs (forward, backward) replayed back to back, events between them"},
        "forward_ms": round(f_ms, 4), "backward_ms": round(b_ms, 4),
        "roofline": {"kernel": "backward pass (4 grouped GEMMs + 5 CUDA-core kernels)", "bound": "tensor",
                     "achieved": round(bwd_tflops, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(bwd_tflops / peak, 4), "traffic": None,
                     "peak_source": f"{pk_kind} {which} (timed region {wall:.2f} s)",
                     "frac_of_sustained_peak": round(bwd_tflops / pk["bf16_tflops_sustained"], 4),
                     "flops": "2 x the forward's grouped-GEMM FLOPs: T(12kDF + 12DFs)"},
        "gpu_launches": (n_fwd + n_bwd) * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    del g_fwd, g_bwd


def run_reference(args, w: mi.Workload, rank: int, world: int):
    """The oracle on the host cores, each step a bounded sample of the workload (rank 0 only)."""
    if rank != 0:
        return
    sample = OracleSample(w, args.weights)
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    steps, done_all, secs_all = [], 0, 0.0
    for s in range(args.warmup + args.steps):
        v, done, elapsed = sample.rate(budget)
        if s >= args.warmup:
            steps.append(v)
            done_all += done
            secs_all += elapsed
    value = statistics.mean(steps)
    ms = w.T / value * 1e3
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "ms_per_step_basis": (f"extrapolated: T = {w.T} tokens / the sampled rate; each timed step ran the oracle "
                              f"on a sample of about {budget:.0f} s ({done_all} tokens in {secs_all:.1f} s over "
                              f"{args.steps} steps), not on all T tokens"),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": w.name, "T": w.T, "D": w.D, "E": w.E, "k": w.k, "F": w.F, "Fs": w.Fs, "bias": w.bias,
                   "weights": "E4M3 codes + per-row fp32 scales" if args.weights == "fp8" else "bf16"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": sample.cores, "kind": "oracle",
                         "sample": f"per step: {sample.describe(done_all // max(1, args.steps), secs_all / max(1, args.steps))}"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    # the default is the largest single-GPU configuration: the DeepSeek-V3-shaped prefill layer
    ap.add_argument("--workload", default="deepseek", choices=sorted(mi.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--train", action="store_true",
                    help="time a training step (forward saving g|u + backward) instead of the forward")
    ap.add_argument("--tiling", default="auto", choices=["auto", "row", "wide", "pair"],
                    help="prefill tiling of the expert GEMMs (bf16): the layer's default, 128-row tiles for both, "
                         "token-wide tiles for both, or token-wide tiles on CTA pairs for both")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="expert weight format; fp8 (E4M3, per-row scales) runs the decode kernels, T <= 64")
    args = ap.parse_args()
    w = mi.WORKLOADS[args.workload]
    if args.weights == "fp8" and w.T > 64:
        ap.error(f"--weights fp8 is the decode path (T <= 64); workload {w.name} has T = {w.T}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank, world)
        return
    import datetime

    import torch.distributed as dist

    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    try:
        if args.train:
            run_train(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
