#!/usr/bin/env python
"""Benchmark of the MoVA value path (router -> grouping -> experts -> combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
    python bench.py --impl reference ...     # the fp64 CPU oracle as the reference arm

A step is one pass of the whole value path over one batch of synthetic tokens
(seeded, see mova_inputs).  The timed region is one CUDA graph holding all K
steps, launched once between a barrier + synchronize on both sides; the expert
weights rotate over several layers (each layer's weights are read once per
step, as in a real forward pass), so the weights a step reads are far larger
than L2.  Per-kernel durations come from stage events recorded inside the
same graph.  Rank 0 prints one JSON line.  Multi-GPU: one process per GPU,
each on its own batch (weak scaling, no collective in the data path).
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
}
DEFAULT_STEPS = {"decode": 2000, "prefill": 300, "skewed": 60, "given": 30, "pr1": 200}
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
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle sample budget")
    a = ap.parse_args(argv)
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

def run_mova(a):
    import torch

    from mixture_value_routing_b200 import api

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_on = init_dist(world, "nccl")
    cfg = MI.WORKLOADS[a.workload]
    T, dtype, mode = cfg["T"], cfg["dtype"], cfg["mode"]
    d, E, k, n = MI.D_MODEL, MI.N_EXPERTS, MI.TOP_K, MI.N_OUT
    L = max(1, a.layers)
    wdt = "f32" if dtype == "f32" else "bf16"

    layers = []
    for l in range(L):
        lay = MI.make_layer(a.seed, l, wv_dtype=wdt, bias=cfg["bias"])
        layers.append((dev_of(lay.Wr, "f32", device), dev_of(lay.br, "f32", device),
                       dev_of(lay.Wv, wdt, device)))
        del lay
    # One batch per layer position; every rank has its own tokens.
    batches = [MI.make_batch(T, rank_batch_seed(a.seed, rank), step=l, dtype=dtype, mode=mode)
               for l in range(L)]
    xs = [dev_of(b.x, dtype, device) for b in batches]
    routing = None
    if mode == "given":
        routing = [(torch.from_numpy(b.idx).to(device), torch.from_numpy(b.w).to(device))
                   for b in batches]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    v = torch.empty((T, n), dtype=tdt, device=device)
    ws = torch.empty(api.workspace_size(T, d, E, k, n), dtype=torch.uint8, device=device)
    path = api.auto_path(T, tdt)

    def step(i, events=None):
        l = i % L
        Wr, br, Wv = layers[l]
        if routing is None:
            api.value_routed(xs[l], Wr, br, Wv, k, MI.SCALE, out=v, ws=ws, events=events)
        else:
            idx, w = routing[l]
            api.value(xs[l], idx, w, Wv, ws=ws, events=events)

    # Distinct experts each layer's step streams (for the decode byte count).
    distinct = []
    for l in range(L):
        if routing is None:
            _, idx_l, _ = api.value_routed(xs[l], *layers[l], k, MI.SCALE, return_routing=True)
        else:
            idx_l = routing[l][0]
        distinct.append(int(torch.unique(idx_l.long()).numel()))

    for i in range(a.warmup):
        step(i)
    torch.cuda.synchronize()

    K = a.steps
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
    # The same K steps with stage events between the kernels: the per-kernel
    # durations.  Events serialise the kernels, so this replay is not the
    # headline number.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for row in evs:  # torch creates the CUDA event on its first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph, stream=cap):
        for i in range(K):
            step(i, events=evs[i])
    torch.cuda.synchronize()
    graph.replay()  # untimed warm-up replays
    pgraph.replay()
    torch.cuda.synchronize()

    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier(dist_on)
    torch.cuda.synchronize()
    with ClockSampler(device) as clk:
        t0.record()
        graph.replay()
        t1.record()
        torch.cuda.synchronize()
    barrier(dist_on)
    ms_local = t0.elapsed_time(t1)
    ms = allmax(ms_local, dist_on, device)
    status, _ = api.get_status(ws)
    assert status == "MOVA_OK", status
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record()
    pgraph.replay()
    p1.record()
    torch.cuda.synchronize()
    prof_ms = p0.elapsed_time(p1)

    stage_ms = {s: 0.0 for s in STAGES}
    for i in range(K):
        for j, s in enumerate(STAGES):
            stage_ms[s] += evs[i][j].elapsed_time(evs[i][j + 1])
    stage_avg_us = {s: 1e3 * stage_ms[s] / K for s in STAGES}
    del graph, pgraph

    peaks, peak_src = load_peaks()
    ms_per_step = ms / K
    value = job_value(world, T, K, ms)

    # Roofline of the dominant kernel (the expert kernel at these sizes).
    xs_b = 2 if dtype == "bf16" else 4
    dom = max(stage_avg_us, key=stage_avg_us.get)
    if path == "stream" or dom != "experts":
        Dm = statistics.mean(distinct)
        expert_bytes = Dm * n * d * xs_b + T * d * xs_b + T * k * n * 4
        alg = {"route": E * d * 4 + E * 4 + T * d * xs_b + T * k * 8,
               "group": 3 * T * k * 4 + (2 * E + 1) * 4,
               "experts": expert_bytes,
               "combine": T * k * n * 4 + T * n * xs_b + T * k * 4}
        dur = stage_avg_us[dom] * 1e-6
        achieved = alg[dom] / dur / 1e9
        peak = float(peaks["hbm_gbs"])
        key = {"experts": "experts_stream"}.get(dom, dom)
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "traffic": ncu_traffic(key, Dm if key == "experts_stream" else 1),
                "algorithmic_bytes_per_launch": int(alg[dom]),
                "peak_source": f"{peak_src} (hbm_gbs, copy)"}
    else:
        flops = 2.0 * T * k * d * n
        dur = stage_avg_us["experts"] * 1e-6
        achieved = flops / dur / 1e12
        peak = float(peaks["bf16_tflops"])
        roof = {"kernel": "experts", "bound": "tensor", "achieved": round(achieved, 1),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": ncu_traffic("experts_tensor", T * k),
                "algorithmic_flops_per_launch": flops,
                "peak_source": f"{peak_src} (bf16_tflops, burst)"}

    # End to end through the public API with host buffers.
    e2e = None
    if not a.no_e2e:
        xh = [torch.empty_like(x, device="cpu").pin_memory() for x in xs]
        for i, x in enumerate(xs):
            xh[i].copy_(x)
        vh = torch.empty((T, n), dtype=tdt).pin_memory()
        xd = torch.empty_like(xs[0])
        Ke = min(K, 500)

        def e2e_step(i):
            l = i % L
            xd.copy_(xh[l], non_blocking=True)
            Wr, br, Wv = layers[l]
            if routing is None:
                out = api.value_routed(xd, Wr, br, Wv, k, MI.SCALE, ws=ws)
            else:
                out = api.value(xd, routing[l][0], routing[l][1], Wv, ws=ws)
            vh.copy_(out, non_blocking=True)

        for i in range(a.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        barrier(dist_on)
        torch.cuda.synchronize()
        e0.record()
        for i in range(Ke):
            e2e_step(i)
        e1.record()
        torch.cuda.synchronize()
        barrier(dist_on)
        ems = allmax(e0.elapsed_time(e1), dist_on, device)
        e2e = {"value": round(job_value(world, T, Ke, ems), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(xs[0].numel() * xs[0].element_size()),
               "d2h_bytes_per_step": int(vh.numel() * vh.element_size()), "steps": Ke,
               "ms_per_step": round(ems / Ke, 5)}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
        "data": "synthetic (seeded; mova_inputs)",
        "config": {"workload": WORKLOAD_TEXT[a.workload], "tokens_per_step_per_gpu": T,
                   "layers_rotated": L, "expert_path": path,
                   "l2": f"weights rotate over {L} layers ({L * E * n * d * xs_b / 1e9:.2f} GB) "
                         f"> 126 MB L2; no flush",
                   "distinct_experts_per_step": distinct, "timing": "one CUDA graph of the K steps, replayed once",
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "stage_us": {s: round(u, 3) for s, u in stage_avg_us.items()},
        "stage_timing": f"second replay of the K steps with stage events ({prof_ms / K * 1e3:.2f} us/step)",
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(a, budget_s=a.cpu_seconds)
    if dist_on:
        import torch.distributed as dist
        dist.destroy_process_group()
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
    if mode == "given":
        return O.combine(x, bat.idx[rows].astype(np.int64), bat.w[rows].astype(np.float64),
                         lay.Wv, wv_dt)
    v, _ = O.value_routed(x, lay.Wr.astype(np.float64), lay.br.astype(np.float64), lay.Wv,
                          MI.TOP_K, MI.SCALE, wv_dt)
    return v


def cpu_baseline(a, budget_s=12.0, steps=None, warmup=0):
    """Time the oracle, as it stands, on seeded batches of the same workload:
    whole steps when they fit the budget, else a sample of tokens per step.
    `warmup` untimed steps (of at most 8 tokens each) run first."""
    from oracle import mova_oracle as O
    cfg = MI.WORKLOADS[a.workload]
    T, dtype, mode = cfg["T"], cfg["dtype"], cfg["mode"]
    wdt = "f32" if dtype == "f32" else "bf16"
    lay = MI.make_layer(a.seed, 0, wv_dtype=wdt, bias=cfg["bias"])
    bat = MI.make_batch(T, a.seed, dtype=dtype, mode=mode)
    # Estimate the per-token cost on a small sample first.
    t = time.perf_counter()
    _oracle_tokens(O, lay, bat, np.arange(min(T, 4)), mode, wdt, dtype)
    per_tok = (time.perf_counter() - t) / min(T, 4)
    if steps is None:
        rows_per = T if per_tok * T <= budget_s / 3 else max(1, int(budget_s / 3 / per_tok))
        nsteps = None
    else:
        rows_per = T if per_tok * T * steps <= budget_s else max(1, int(budget_s / steps / per_tok))
        nsteps = steps
    rng = np.random.default_rng(1234)
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
        if (nsteps is not None and i >= nsteps) or (nsteps is None and el >= budget_s):
            break
    el = time.perf_counter() - t0
    return {"value": round(done / el, 3), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"{i} oracle steps of {rows_per} of the {T} tokens of a seeded "
                      f"{a.workload} batch ({done} tokens, {el:.1f} s, numpy fp64)"
                      + (f", after {warmup} untimed warm-up steps of up to 8 tokens" if warmup else ""),
            "steps_timed": i, "seconds": round(el, 2)}


def run_reference(a):
    rank, _, world = dist_env()
    if rank != 0:
        return
    budget = 150.0
    cb = cpu_baseline(a, budget_s=budget, steps=a.steps, warmup=a.warmup)
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "tokens/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": round(1e3 * cb["seconds"] / max(1, cb["steps_timed"]), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded; mova_inputs)",
            "config": {"workload": WORKLOAD_TEXT[a.workload]},
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
