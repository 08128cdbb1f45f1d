#!/usr/bin/env python
"""Benchmark of the MoVA value path (router -> grouping -> experts -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
    python bench.py --impl reference ...     # the fp64 CPU oracle as the reference arm

A step is one pass of the whole value path over one batch of synthetic tokens
(seeded, see mova_inputs).  The timed region is one CUDA graph holding all K
steps, launched once between a barrier + synchronize on both sides (a short
spin kernel before the start event hides the host's submission of the graph,
so the events bracket only the K steps' device work); the expert
weights rotate over several layers (each layer's weights are read once per
step, as in a real forward pass), so the weights a step reads are far larger
than L2.  Per-kernel durations come from a second replay with stage events
recorded inside the graph, less the measured cost of an empty event pair.
Rank 0 prints one JSON line: the headline workload (--workload, decode T=8 by
default) and, as sub-records of the same line, the other workloads of the
metric and scope (--also: prefill T=4096, skewed prefill T=16384,
routing-given L=32768, attend), each with its own steps, roofline, end-to-end
rate and CPU baseline; `config` describes the workload (the same on the
reference arm's line), `run` what the run measured.  Multi-GPU: one process per GPU, each on its own batch (weak
scaling, no collective in the data path).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mova_inputs as MI  # noqa: E402

WORKLOAD_TEXT = {
    "decode": "decode step T=8 (d=2560, 64 experts of 2560->1024, top-4, bf16 x/experts, fp32 router)",
    "prefill": "prefill T=4096 (d=2560, 64 experts of 2560->1024, top-4, bf16 x/experts, fp32 router)",
    "skewed": "skewed prefill T=16384 (router bias 2 ln Zipf(1.2); otherwise as prefill)",
    "given": "routing-given recompute L=32768 (int8 top-4 indices, fp16 Dirichlet(1)x2.5 weights)",
    "pr1": "PR1 reference T=128, all fp32",
    "attend": "attend: one query token's 32 heads over L=32768 cached positions, values recomputed from the "
              "compact cache (int8 top-4, fp16 weights) inside the PV product, never stored",
}
DEFAULT_STEPS = {"decode": 2000, "prefill": 300, "skewed": 60, "given": 30, "pr1": 200, "attend": 30}
METRIC = "MoVA value-path tokens/s at T=8 & T=4096; % of HBM / bf16 tensor roofline"
STAGES = ("route", "group", "experts", "combine")
KERNEL_SOURCES = {
    "route": ["router.cu"], "group": ["permute.cu"],
    "experts_stream": ["stream_experts.cu", "sm100.cuh", "route_select.cuh"],
    "experts_tensor": ["grouped_gemm_pair.cu", "sm100.cuh"], "combine": ["combine.cu"],
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("mova", "reference"), default="mova")
    ap.add_argument("--workload", choices=tuple(WORKLOAD_TEXT), default="decode")
    ap.add_argument("--layers", type=int, default=4, help="weight sets rotated over the steps")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=8.0, help="oracle sample budget")
    ap.add_argument("--also", default="prefill,skewed,given,attend",
                    help="workloads measured as sub-records of the same line (comma list; '=' for none)")
    a = ap.parse_args(argv)
    a.also = [w for w in a.also.split(",") if w and w != "="]
    for w in a.also:
        if w not in WORKLOAD_TEXT:
            ap.error(f"--also: unknown workload {w}")
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


# ---------------------------------------------------------------------------
# Process group
# ---------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world > 1


def rank_batch_seed(seed, rank):
    """Each rank draws its own tokens; every rank holds the same layer weights."""
    return seed + 7919 * rank


def job_value(world, tokens_per_rank_step, steps, ms_max):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank_step * steps / (ms_max / 1e3)


def barrier(on):
    if on:
        import torch.distributed as dist
        dist.barrier()


def allmax(value, on, device):
    if not on:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# Clocks during the timed region (NVML, sampled in a thread)
# ---------------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device, period_s=0.002):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml as N
            N.nvmlInit()
            self.N = N
            h = None
            try:
                import torch
                p = torch.cuda.get_device_properties(torch_device)
                bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
                h = N.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                h = N.nvmlDeviceGetHandleByIndex(0)
            self.h = h
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that
            self.err = str(e)

    def _reasons(self):
        N = self.N
        fn = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            N.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        N = self.N
        while not self._stop.is_set():
            try:
                self.samples.append((N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM),
                                     self._reasons(),
                                     N.nvmlDeviceGetUtilizationRates(self.h).gpu))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": f"NVML unavailable: {getattr(self, 'err', '')}"}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        mhz = [s[0] for s in busy]
        mask = 0
        for s in busy:
            mask |= s[1]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": [name for bit, name in _REASONS.items() if mask & bit and bit != 0x1],
                "samples": len(busy)}


# ---------------------------------------------------------------------------
# Inputs on the device
# ---------------------------------------------------------------------------

def bf16_dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def dev_of(a, dtype, device):
    import torch
    if dtype == "bf16":
        return bf16_dev(a, device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(files):
    h = hashlib.sha256()
    for name in files + ["common.cuh"]:
        p = os.path.join(ROOT, "mixture_value_routing_b200", "csrc", name)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, units_per_launch):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(kernel_key)
    if not rec or rec.get("src_sha") != source_sha(KERNEL_SOURCES[kernel_key]):
        return None
    return rec["dram_bytes_per_unit"] * units_per_launch


# ---------------------------------------------------------------------------
# The CUDA arm
# ---------------------------------------------------------------------------

class _Layers:
    """The L rotated layers' weights on the device (shared by the workloads;
    the skewed workload swaps in its Zipf router bias)."""

    def __init__(self, a, device, wdt):
        self.L = max(1, a.layers)
        self.items = []
        for l in range(self.L):
            lay = MI.make_layer(a.seed, l, wv_dtype=wdt)
            self.items.append((dev_of(lay.Wr, "f32", device), dev_of(lay.br, "f32", device),
                               dev_of(lay.Wv, wdt, device)))
            del lay
        self.zipf = dev_of(MI.zipf_bias(), "f32", device)

    def get(self, l, bias):
        Wr, br, Wv = self.items[l % self.L]
        return Wr, (self.zipf if bias == "zipf" else br), Wv


def _replay_for(graph, seconds, step_s, K):
    """Replay `graph` (K steps) back to back for about `seconds` (untimed
    load around the timed replay, so that the clock sampler sees the GPU
    under the same load)."""
    import torch
    reps = max(1, int(seconds / max(step_s * K, 1e-6)))
    for _ in range(reps):
        graph.replay()
    torch.cuda.synchronize()
    return reps


# About 2 ms of spinning at the B200's clocks: longer than the host takes to
# record an event and submit the largest timed graph.
COVER_CYCLES = 4_000_000


def _cover_submission():
    """Keep the stream busy while the host records the start event and
    submits the timed graph: the start event then fires only when the spin
    ends, with the graph's kernels already queued, so the timed region holds
    the K steps' device work and not the host's submission latency (which
    otherwise adds tens of microseconds to a region of a few hundred)."""
    import torch
    torch.cuda._sleep(COVER_CYCLES)


def workload_config(a, name, world):
    """The `config` of a workload's record: what the workload is and how L2 is
    kept from serving the weights, the same on the reference arm's line as on
    this one.  What a run measured (the routing's expert counts) and how it
    was timed go under the record's "run" key."""
    cfg = MI.WORKLOADS[name]
    T, xs_b = cfg["T"], 2 if cfg["dtype"] == "bf16" else 4
    L, d, E, n = max(1, a.layers), MI.D_MODEL, MI.N_EXPERTS, MI.N_OUT
    return {"workload": WORKLOAD_TEXT[name], "tokens_per_step_per_gpu": T, "layers_rotated": L,
            "l2": f"weights rotate over {L} layers ({L * E * n * d * xs_b / 1e9:.2f} GB) > 126 MB L2; no flush",
            "parallelism": f"dp{world} (independent batches, no collective)"}


def measure_workload(a, name, K, layers, device, dist_on, world, rank, peaks, peak_src):
    """One workload: W warm-up steps, then exactly K steps in one CUDA graph
    timed with CUDA events between barrier + synchronize (max over ranks);
    per-kernel durations from a second replay with stage events; the
    end-to-end rate through the Python API with host buffers."""
    import torch

    from mixture_value_routing_b200 import api

    cfg = MI.WORKLOADS[name]
    T, dtype, mode = cfg["T"], cfg["dtype"], cfg["mode"]
    d, E, k, n = MI.D_MODEL, MI.N_EXPERTS, MI.TOP_K, MI.N_OUT
    L = layers.L
    xs_b = 2 if dtype == "bf16" else 4
    batches = [MI.make_batch(T, rank_batch_seed(a.seed, rank), step=l, dtype=dtype, mode=mode)
               for l in range(L)]
    xs = [dev_of(b.x, dtype, device) for b in batches]
    routing = None
    if mode in ("given", "attend"):
        routing = [(torch.from_numpy(b.idx).to(device), torch.from_numpy(b.w).to(device))
                   for b in batches]
    probs = [torch.from_numpy(b.probs).to(device) for b in batches] if mode == "attend" else None
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    v = torch.empty((T, n), dtype=tdt, device=device)
    if mode == "attend":
        ws = torch.empty(api.attend_workspace_size(T, d, E, k, n, MI.ATTEND_HEADS), dtype=torch.uint8,
                         device=device)
    else:
        ws = torch.empty(api.workspace_size(T, d, E, k, n), dtype=torch.uint8, device=device)
    path = api.auto_path(T, tdt)

    def step(i, events=None):
        l = i % L
        Wr, br, Wv = layers.get(l, cfg["bias"])
        if routing is None:
            api.value_routed(xs[l], Wr, br, Wv, k, MI.SCALE, out=v, ws=ws, events=events)
        elif probs is not None:
            # mova_value_attend takes no stage events: the step is timed whole.
            idx, w = routing[l]
            api.value_attend(xs[l], idx, w, Wv, probs[l], ws=ws)
        else:
            idx, w = routing[l]
            api.value(xs[l], idx, w, Wv, ws=ws, events=events)

    # Distinct experts each layer's step streams, the busiest expert's load,
    # and the first step's loads of its active experts (descending).
    distinct, max_load, loads0 = [], [], []
    for l in range(L):
        if routing is None:
            _, idx_l, _ = api.value_routed(xs[l], *layers.get(l, cfg["bias"]), k, MI.SCALE,
                                           return_routing=True)
        else:
            idx_l = routing[l][0]
        cnt = torch.bincount(idx_l.long().flatten(), minlength=E)
        distinct.append(int((cnt > 0).sum().item()))
        max_load.append(int(cnt.max().item()))
        if l == 0:
            loads0 = sorted((int(c) for c in cnt.tolist() if c > 0), reverse=True)

    for i in range(a.warmup):
        step(i)
    torch.cuda.synchronize()

    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    # The timed graph: K steps back to back, nothing between the kernels (so
    # programmatic dependent launch can overlap each kernel's launch with its
    # predecessor).
    graph = torch.cuda.CUDAGraph()
    launches0 = api.launch_count()
    with torch.cuda.graph(graph, stream=cap):
        for i in range(K):
            step(i)
    launches = api.launch_count() - launches0  # kernels the timed graph holds
    # The same K steps with stage events between the kernels, plus one empty
    # event pair per step: stage events serialise the kernels and each event
    # node costs time of its own, which the empty pair measures.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    empty = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
    for row in evs + empty:  # torch creates the CUDA event on its first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=cap):
        for i in range(K):
            step(i, events=evs[i])
            empty[i][0].record()
            empty[i][1].record()
    torch.cuda.synchronize()
    graph.replay()  # untimed warm-up replays
    pgraph.replay()
    torch.cuda.synchronize()

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    w0 = time.perf_counter()
    graph.replay()
    torch.cuda.synchronize()
    est_step_s = (time.perf_counter() - w0) / K
    with ClockSampler(device) as clk:
        _replay_for(graph, 0.25, est_step_s, K)
        barrier(dist_on)
        torch.cuda.synchronize()
        _cover_submission()
        t0.record()
        graph.replay()
        t1.record()
        torch.cuda.synchronize()
        barrier(dist_on)
        _replay_for(graph, 0.25, est_step_s, K)
    ms_local = t0.elapsed_time(t1)
    ms = allmax(ms_local, dist_on, device)
    status, _ = api.get_status(ws)
    assert status == "MOVA_OK", status
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    _cover_submission()
    p0.record()
    pgraph.replay()
    p1.record()
    torch.cuda.synchronize()
    prof_ms = p0.elapsed_time(p1)
    stage_ms = {s: 0.0 for s in STAGES}
    empty_ms = 0.0
    for i in range(K):
        for j, s in enumerate(STAGES):
            stage_ms[s] += evs[i][j].elapsed_time(evs[i][j + 1])
        empty_ms += empty[i][0].elapsed_time(empty[i][1])
    stage_avg_us = {s: 1e3 * stage_ms[s] / K for s in STAGES}
    empty_us = 1e3 * empty_ms / K
    del graph, pgraph

    ms_per_step = ms / K
    if mode == "attend":
        # No stage events: the whole step (coefficients, grouping, gather,
        # GEMM with the attend epilogue, reduction) stands for the experts.
        stage_avg_us = {s: 0.0 for s in STAGES}
        stage_avg_us["experts"] = 1e3 * ms_per_step
        empty_us = 0.0
    value = job_value(world, T, K, ms)
    roof = roofline(name, path, T, d, E, k, n, xs_b, distinct, stage_avg_us, empty_us, ms_per_step,
                    peaks, peak_src)
    if mode == "attend":
        roof["kernel"] = "whole attend step (no stage events in mova_value_attend)"
        roof["traffic"] = None

    e2e = None
    if not a.no_e2e:
        e2e = measure_e2e(a, T, L, xs, routing, layers, cfg, v, ws, k, n, tdt, dist_on, world, device, probs)

    rec = {
        "value": round(value, 1), "unit": "tokens/s", "steps": K, "warmup": a.warmup,
        "ms_per_step": round(ms_per_step, 5), "dtype": dtype,
        "config": workload_config(a, name, world),
        "run": {"expert_path": path, "distinct_experts_per_step": distinct,
                "max_expert_load_per_step": max_load, "expert_loads_first_step": loads0,
                "timing": "one CUDA graph of the K steps, replayed once between barrier + "
                          "synchronize; CUDA events on the replaying stream"},
        "stage_us": {s: round(u, 3) for s, u in stage_avg_us.items()},
        "event_pair_us": round(empty_us, 3),
        "stage_timing": f"second replay of the K steps with stage events ({prof_ms / K * 1e3:.2f} us/step); "
                        f"a kernel's duration = its stage time minus the measured empty event pair",
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": dict(clk.summary(), window="sampled from 0.25 s of the same graph replayed before "
                                             "the timed replay, through it, to 0.25 s after"),
    }
    return rec


def roofline(name, path, T, d, E, k, n, xs_b, distinct, stage_us, empty_us, ms_per_step, peaks,
             peak_src):
    """Roofline of the dominant kernel (duration = stage time minus the event
    pair) and of the whole step (duration = ms_per_step)."""
    Dm = statistics.mean(distinct)
    dom = max(stage_us, key=stage_us.get)
    dur_us = max(stage_us[dom] - empty_us, 1e-3)
    if path == "stream":
        kernel_bytes = Dm * n * d * xs_b + T * d * xs_b + T * n * xs_b
        step_bytes = Dm * n * d * xs_b + E * d * 4 + E * 4 + T * d * xs_b + T * n * xs_b
        peak = float(peaks["hbm_gbs"])
        achieved = kernel_bytes / (dur_us * 1e-6) / 1e9
        step_achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
        key = "experts_stream"
        return {"kernel": "stream_experts_kernel (route, group, stream, combine)" if dom == "experts" else dom,
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "frac_of_nominal_8000": round(achieved / 8000.0, 4),
                "traffic": ncu_traffic(key, Dm) if dom == "experts" else None,
                "kernel_us": round(dur_us, 3),
                "algorithmic_bytes_per_launch": int(kernel_bytes),
                "step": {"achieved": round(step_achieved, 1), "frac": round(step_achieved / peak, 4),
                         "frac_of_nominal_8000": round(step_achieved / 8000.0, 4),
                         "algorithmic_bytes_per_step": int(step_bytes)},
                "peak_source": f"{peak_src} (hbm_gbs, copy)"}
    flops = 2.0 * T * k * d * n
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (dur_us * 1e-6) / 1e12
    step_achieved = flops / (ms_per_step * 1e-3) / 1e12
    return {"kernel": "grouped_gemm_pair_kernel" if dom == "experts" else dom,
            "bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "frac_of_nominal_2250": round(achieved / 2250.0, 4),
            "traffic": ncu_traffic("experts_tensor", T * k) if dom == "experts" else None,
            "kernel_us": round(dur_us, 3), "algorithmic_flops_per_launch": flops,
            "step": {"achieved": round(step_achieved, 1), "frac": round(step_achieved / peak, 4),
                     "frac_of_nominal_2250": round(step_achieved / 2250.0, 4)},
            "peak_source": f"{peak_src} (bf16_tflops, burst)"}


def measure_e2e(a, T, L, xs, routing, layers, cfg, v, ws, k, n, tdt, dist_on, world, device, probs=None):
    """The same metric through the C ABI's host-buffer calls (mova_value_routed_host,
    mova_value_host, mova_value_attend_host): every step copies its inputs from
    pinned host memory (x; the stored int8 indices and fp16 weights in
    routing-given and attend mode; the attention probabilities in attend mode)
    into the device workspace, runs the path, and copies v (o in attend mode)
    back to pinned host memory.  Two steps are in flight, on two streams with a
    workspace each, so that one step's copies overlap the other's kernels."""
    import torch

    from mixture_value_routing_b200 import api
    xh = [x.cpu().pin_memory() for x in xs]
    rh = None if routing is None else [(i.cpu().pin_memory(), w.cpu().pin_memory()) for i, w in routing]
    ph = None if probs is None else [p.cpu().pin_memory() for p in probs]
    d = xs[0].shape[1]
    E = layers.get(0, cfg["bias"])[2].shape[0]
    if ph is not None:
        H = probs[0].shape[0]
        nbytes = api.attend_workspace_size_host(T, d, E, k, n, H)
        outs = [torch.empty((H, 128), dtype=torch.float32).pin_memory() for _ in range(2)]
    else:
        nbytes = api.workspace_size_host(T, d, E, k, n)
        outs = [torch.empty((T, n), dtype=tdt).pin_memory() for _ in range(2)]
    wss = [torch.empty(nbytes, dtype=torch.uint8, device=device) for _ in range(2)]
    streams = [torch.cuda.Stream(device) for _ in range(2)]
    Ke = max(3, min(500, int(0.2 / max(1e-6, 2.5e-8 * T * 20))))

    def e2e_step(i):
        l, j = i % L, i % 2
        Wr, br, Wv = layers.get(l, cfg["bias"])
        if rh is None:
            api.value_routed_host(xh[l], Wr, br, Wv, k, MI.SCALE, out=outs[j], ws=wss[j], stream=streams[j])
        elif ph is None:
            api.value_host(xh[l], rh[l][0], rh[l][1], Wv, out=outs[j], ws=wss[j], stream=streams[j])
        else:
            api.value_attend_host(xh[l], rh[l][0], rh[l][1], Wv, ph[l], out=outs[j], ws=wss[j],
                                  stream=streams[j])

    for i in range(a.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist_on)
    torch.cuda.synchronize()
    e0.record(cur)
    for s in streams:
        s.wait_event(e0)
    for i in range(Ke):
        e2e_step(i)
    for s in streams:
        cur.wait_stream(s)
    e1.record(cur)
    torch.cuda.synchronize()
    barrier(dist_on)
    ems = allmax(e0.elapsed_time(e1), dist_on, device)
    h2d = xs[0].numel() * xs[0].element_size()
    if routing is not None:
        h2d += sum(t.numel() * t.element_size() for t in routing[0])
    if probs is not None:
        h2d += probs[0].numel() * probs[0].element_size()
    return {"value": round(job_value(world, T, Ke, ems), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(outs[0].numel() * outs[0].element_size()),
            "steps": Ke, "ms_per_step": round(ems / Ke, 5),
            "api": "C-ABI host-buffer calls; two steps in flight on two streams"}


def run_mova(a):
    import torch

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_on = init_dist(world, "nccl")
    peaks, peak_src = load_peaks()
    head = a.workload
    wdt = "f32" if MI.WORKLOADS[head]["dtype"] == "f32" else "bf16"
    layers = _Layers(a, device, wdt)
    # The headline workload with --steps; the other workloads of the metric
    # and of the scope (prefill, skewed prefill, routing-given recompute) as
    # sub-records of the same line, each with its own step count.
    extras = [w for w in a.also if w != head and MI.WORKLOADS[w]["dtype"] == MI.WORKLOADS[head]["dtype"]]
    recs = {}
    for name in [head] + extras:
        K = a.steps if name == head else DEFAULT_STEPS[name]
        recs[name] = measure_workload(a, name, K, layers, device, dist_on, world, rank, peaks, peak_src)
        if rank == 0 and world == 1 and not a.no_cpu_baseline:
            budget = a.cpu_seconds if name == head or name == "prefill" else a.cpu_seconds / 2
            recs[name]["cpu_baseline"] = cpu_baseline(a, name, budget_s=budget)
    if dist_on:
        import torch.distributed as dist
        dist.destroy_process_group()
    h = recs[head]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": h["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": h["dtype"],
        "data": "synthetic (seeded; mova_inputs)",
        "config": h["config"], "run": h["run"],
        "stage_us": h["stage_us"], "event_pair_us": h["event_pair_us"], "stage_timing": h["stage_timing"],
        "roofline": h["roofline"], "e2e": h["e2e"], "gpu_launches": h["gpu_launches"], "clocks": h["clocks"],
    }
    if "cpu_baseline" in h:
        line["cpu_baseline"] = h["cpu_baseline"]
    for name in extras:
        line[name] = recs[name]
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# The oracle on the host (CPU baseline / reference arm)
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def _oracle_tokens(O, lay, bat, rows, mode, wv_dt, dtype):
    x = O.to_f64(bat.x[rows], dtype)
    if mode == "attend":
        return O.attend(x, bat.idx[rows].astype(np.int64), bat.w[rows].astype(np.float64), lay.Wv,
                        bat.probs[:, rows].astype(np.float64), wv_dt)
    if mode == "given":
        return O.combine(x, bat.idx[rows].astype(np.int64), bat.w[rows].astype(np.float64),
                         lay.Wv, wv_dt)
    v, _ = O.value_routed(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), lay.Wv,
                          MI.TOP_K, MI.SCALE, wv_dt)
    return v


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _oracle_rate(O, lay, bat, T, mode, wdt, dtype, budget_s, steps, warmup, rows_per, rng):
    """Tokens/s of the oracle over seeded token samples (whole steps when
    rows_per == T); runs `steps` steps, or until `budget_s` when steps is None."""
    for _ in range(warmup):
        _oracle_tokens(O, lay, bat, np.arange(min(T, rows_per, 8)), mode, wdt, dtype)
    done = 0
    i = 0
    t0 = time.perf_counter()
    while True:
        rows = np.arange(T) if rows_per >= T else np.sort(rng.choice(T, rows_per, replace=False))
        _oracle_tokens(O, lay, bat, rows, mode, wdt, dtype)
        done += rows.size
        i += 1
        el = time.perf_counter() - t0
        if (steps is not None and i >= steps) or (steps is None and el >= budget_s):
            break
    el = time.perf_counter() - t0
    return done / el, i, done, el


def cpu_baseline(a, name=None, budget_s=8.0, steps=None, warmup=0, one_core=True):
    """Time the oracle, as it stands, on seeded batches of a workload: whole
    steps when they fit the budget, else a seeded sample of tokens per step;
    on all the BLAS threads, then (one_core) on one.  `warmup` untimed steps
    (of at most 8 tokens each) run first."""
    from oracle import mova_oracle as O
    name = name or a.workload
    cfg = MI.WORKLOADS[name]
    T, dtype, mode = cfg["T"], cfg["dtype"], cfg["mode"]
    wdt = "f32" if dtype == "f32" else "bf16"
    lay = MI.make_layer(a.seed, 0, wv_dtype=wdt, bias=cfg["bias"])
    bat = MI.make_batch(T, a.seed, dtype=dtype, mode=mode)
    # Estimate the per-token cost on a small sample first.
    t = time.perf_counter()
    _oracle_tokens(O, lay, bat, np.arange(min(T, 4)), mode, wdt, dtype)
    per_tok = (time.perf_counter() - t) / min(T, 4)
    share = budget_s / 2 if one_core else budget_s
    if steps is None:
        rows_per = T if per_tok * T <= share / 3 else max(1, int(share / 3 / per_tok))
    else:
        rows_per = T if per_tok * T * steps <= share else max(1, int(share / steps / per_tok))
    rate, i, done, el = _oracle_rate(O, lay, bat, T, mode, wdt, dtype, share, steps, warmup, rows_per,
                                     np.random.default_rng(1234))
    out = {"value": round(rate, 3), "unit": "tokens/s", "cores": _blas_threads(),
           "cpu_model": _cpu_model(), "host_cpus": os.cpu_count(),
           "kind": "oracle",
           "sample": f"{i} oracle steps of {rows_per} of the {T} tokens of a seeded "
                     f"{name} batch ({done} tokens, {el:.1f} s, numpy fp64)"
                     + (f", after {warmup} untimed warm-up steps of up to 8 tokens" if warmup else ""),
           "steps_timed": i, "seconds": round(el, 2)}
    if one_core:
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                r1, i1, d1, e1 = _oracle_rate(O, lay, bat, T, mode, wdt, dtype, share, None, 0,
                                              rows_per, np.random.default_rng(4321))
            out["one_core"] = {"value": round(r1, 3), "unit": "tokens/s", "cores": 1,
                               "sample": f"{i1} oracle steps of {rows_per} tokens ({d1} tokens, {e1:.1f} s)"}
        except Exception as e:  # threadpoolctl unavailable: say so
            out["one_core"] = {"value": None, "note": f"not measured: {e}"}
    return out


def run_reference(a):
    rank, _, world = dist_env()
    if rank != 0:
        return
    budget = 150.0
    cb = cpu_baseline(a, a.workload, budget_s=budget, steps=a.steps, warmup=a.warmup, one_core=False)
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(1e3 * cb["seconds"] / max(1, cb["steps_timed"]), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded; mova_inputs)",
            "config": workload_config(a, a.workload, world),
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    a = parse(argv)
    if a.impl == "reference":
        run_reference(a)
    else:
        run_mova(a)


if __name__ == "__main__":
    main()
