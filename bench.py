#!/usr/bin/env python
"""Benchmark of the decode-time MoE layer with batch-aware expert re-routing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload q30b_b16_oea4] [--no-extra]

One step = one moe_layer_decode call (router GEMV + softmax + top-k,
re-selection + token lists, grouped SwiGLU expert FFN with the weighted
combine) on one decode batch, inputs resident in HBM.  Weights rotate over
4 identical copies (each larger than the 126 MB L2) so no step reads
weights another step left in L2.  Steps run as CUDA-graph replays of 4
consecutive layer calls (one per copy); the graph keeps every kernel of
every call.

Printed (rank 0, one JSON line): value = algorithmic bytes of all ranks per
second (activated experts x 3 d d_ff x 2 B + router weights + x + y), the
roofline of the dominant kernel (up to 64 tokens the fused layer kernel,
which is the whole call; above, the expert kernel, timed with events
around moe_expert_ffn), the oracle
timed on the host cores (cpu_baseline), an end-to-end number through the
Python API with host buffers (e2e), and the SM clocks sampled with NVML
during the timed region.

N > 1 (torchrun): every rank runs an independent replica of the layer on
its own GPU (the layer is single-GPU; there is no data-path collective);
timing is the max over ranks; scaling is weak.

--impl reference times the CPU oracle on the host cores instead (rank 0
only), each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_synth as ms  # noqa: E402

METRIC = "MoE-layer decode µs & achieved HBM GB/s (% of roofline) vs batch size"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
ROTATE = 4

WORKLOADS = {
    "q30b_b16_oea4": dict(shape="q30b", B=16, mode=1, k0=4, budget=0, rule="OEA k0=4"),
    # up to 8 tokens and 32 activated experts: the warp-MMA expert stream
    "q30b_b4_oea4": dict(shape="q30b", B=4, mode=1, k0=4, budget=0, rule="OEA k0=4"),
    "q30b_b16_none": dict(shape="q30b", B=16, mode=0, k0=0, budget=0, rule="NONE (standard top-8)"),
    "q30b_b64_oea4": dict(shape="q30b", B=64, mode=1, k0=4, budget=0, rule="OEA k0=4"),
    "q30b_b96_oea4": dict(shape="q30b", B=96, mode=1, k0=4, budget=0, rule="OEA k0=4"),
    "q235b_b16_oea4": dict(shape="q235b", B=16, mode=1, k0=4, budget=0, rule="OEA k0=4"),
    "spec_xshare32": dict(shape="q30b", B=32, mode=2, k0=0, budget=32, rule="XShare budget=32",
                          kind="spec"),
    "q30b_b16_affinity": dict(shape="q30b", B=16, mode=3, k0=0, budget=0, rule="Lynx affinity binning"),
    "spec_xshare_hier32": dict(shape="q30b", B=32, mode=4, k0=0, budget=32, group=4, kind="spec",
                               rule="hierarchical XShare budget=32, 4 tokens per request"),
    # per-token channel top-k inside the activated experts (c = 13 % of
    # d_ff, scores drawn at random per (token, slot))
    "q30b_b1_oea4_ch13": dict(shape="q30b", B=1, mode=1, k0=4, budget=0, channels=0.13,
                              rule="OEA k0=4, channel top-k 13 %"),
    "q30b_b4_oea4_ch13": dict(shape="q30b", B=4, mode=1, k0=4, budget=0, channels=0.13,
                              rule="OEA k0=4, channel top-k 13 %"),
}

# DRAM bytes (read + write) per launch of the dominant kernel (the fused
# layer kernel up to 64 tokens) from an ncu capture of the same workload on
# one weight copy (profiles/layer_kernel_q30b_b16_oea4.md, ..._b64_...);
# a workload without an entry reports null.  Entries are dropped whenever
# the kernel changes.
NCU_TRAFFIC = {
    "q30b_b16_oea4": 142883840 + 3248896,
    "q30b_b64_oea4": 284837120 + 4763904,
    # channel top-k workloads: channel_stream_kernel, which moves the weights
    # (profiles/channel_stream_kernel_q30b_oea4_ch13.md)
    "q30b_b1_oea4_ch13": 4969984,
    "q30b_b4_oea4_ch13": 33603328,
}


def workload_desc(w: dict) -> str:
    S = ms.SHAPES[w["shape"]]
    name = {"q30b": "Qwen3-30B-A3B-shaped", "q235b": "Qwen3-235B-A22B-shaped"}[w["shape"]]
    extra = ", speculative batch of 8 requests x 4 drafts" if w.get("kind") == "spec" else ""
    return (f"{name} MoE layer (d={S.d}, E={S.E}, k={S.k}, d_ff={S.F}, bf16 experts), "
            f"decode batch B={w['B']}{extra}, {w['rule']}")


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(S, B, n_active):
    experts = n_active * 3 * S.d * S.F * 2
    router = S.E * S.d * 4 + S.E * 4
    io = B * S.d * 4 * 2
    return experts + router + io, experts + io


# ------------------------------------------------------ multi-rank host --
def max_over_ranks(v: float, world: int, device=None) -> float:
    """Max of a per-rank timing over all ranks (every rank must call it)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    tv = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(tv, op=dist.ReduceOp.MAX)
    return float(tv.item())


def aggregate_gbs(bytes_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """Whole-job GB/s: every rank moves the same bytes per step; the step
    time is the max over ranks."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------- clocks --
class ClockSampler:
    """Polls SM clock and clock-event reasons with NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ----------------------------------------------------------- reference --
def run_reference(args, w, rank):
    import oracle
    if rank != 0:
        return
    S = ms.SHAPES[w["shape"]]
    L = ms.make_weights(S, 0)
    x = ms.make_tokens(S, w["B"], 0, kind=w.get("kind", "normal"))
    cores = len(os.sched_getaffinity(0))
    r0 = oracle.layer(x, L, S.k, w["mode"], w["k0"], w["budget"], group=w.get("group", 1),
                      rows=np.arange(1, dtype=np.int32),
                      threads=cores)
    n_active = r0["lists"]["n_active"]
    total_bytes, _ = algorithmic_bytes(S, w["B"], n_active)
    # size one step: route + re-select the whole batch, FFN for `rows` tokens
    t0 = time.perf_counter()
    oracle.layer(x, L, S.k, w["mode"], w["k0"], w["budget"], group=w.get("group", 1),
                 rows=np.arange(1, dtype=np.int32), threads=cores)
    t_one = time.perf_counter() - t0
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    rows = int(max(1, min(w["B"], budget_s / max(t_one, 1e-6))))
    sel = np.arange(rows, dtype=np.int32)

    def step():
        oracle.layer(x, L, S.k, w["mode"], w["k0"], w["budget"], group=w.get("group", 1), rows=sel, threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = total_bytes * rows / w["B"] / dt / 1e9
    sample = (f"per step: router + {w['rule']} for all {w['B']} tokens, expert FFN for {rows} of "
              f"{w['B']} tokens; bytes scaled by {rows}/{w['B']}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(w), "n_active": n_active},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, S, L, x, seconds=12.0):
    import oracle
    cores = len(os.sched_getaffinity(0))
    n = 0
    t0 = time.perf_counter()
    nact = None
    while True:
        r = oracle.layer(x, L, S.k, w["mode"], w["k0"], w["budget"], group=w.get("group", 1), threads=cores)
        nact = r["lists"]["n_active"]
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = (time.perf_counter() - t0) / n
    total, _ = algorithmic_bytes(S, w["B"], nact)
    return {"value": total / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{n} full layer calls (all {w['B']} tokens), {dt * 1e3:.1f} ms each"}


# ---------------------------------------------------------------- ours --
def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import aware_expert_routing_moe_b200 as moe

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    moe.load_library()
    S = ms.SHAPES[w["shape"]]
    B, mode, k0, budget = w["B"], w["mode"], w["k0"], w["budget"]
    group = w.get("group", 1)
    L = ms.make_weights(S, 0)
    x_np = ms.make_tokens(S, B, 0, kind=w.get("kind", "normal"))
    t = lambda a: torch.from_numpy(a).to(dev)
    Wg, bias = t(L["Wg"]), t(L["bias"])
    # every rotation has its own copy of all layer weights (router included)
    copies = [(t(L["Wgate"].view(np.int16)), t(L["Wup"].view(np.int16)), t(L["Wdown"].view(np.int16)), Wg)]
    for _ in range(ROTATE - 1):
        copies.append(tuple(c.clone() for c in copies[0]))
    x = t(x_np)
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F, dev)
    y = torch.empty(B, S.d, dtype=torch.float32, device=dev)
    nact_t = torch.zeros(4, dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(dev)
    # the copies and the zero-filled workspace were written on the default
    # stream: the calls on s must not start before they are complete
    s.wait_stream(torch.cuda.current_stream(dev))

    def layer(r):
        g, u, dn, wg = copies[r]
        moe.moe_layer_decode(x, wg, bias, g, u, dn, S.k, mode, k0, budget, ws=ws, y=y, n_active=nact_t,
                             group=group)

    with torch.cuda.stream(s):
        for r in range(ROTATE):
            layer(r)
    s.synchronize()
    if moe.moe_check_error(ws, s) != 0:
        raise RuntimeError("device error word set during warm-up")
    n_active = int(nact_t[0].item())
    total_bytes, ffn_bytes = algorithmic_bytes(S, B, n_active)

    # CUDA graphs: one with ROTATE consecutive layer calls, and single calls
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all, stream=s):
        for r in range(ROTATE):
            layer(r)
    g_one = []
    for r in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            layer(r)
        g_one.append(g)

    def replay(nsteps):
        full, rest = divmod(nsteps, ROTATE)
        for _ in range(full):
            g_all.replay()
        for r in range(rest):
            g_one[r].replay()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])

    def timed(fn, nsteps, sampler=None):
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            fn(nsteps)
            e1.record(s)
        e1.synchronize()
        torch.cuda.synchronize(dev)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)  # ms, all steps

    # ---- main timed region: K graph-replayed layer calls.  The clock
    # sampler runs from the warm-up through the last leg below, so that a
    # short timed region still gets a clock record of several samples; the
    # GPU is busy with the same kernels throughout.
    sampler = ClockSampler(local_rank)
    sampler.__enter__()
    with torch.cuda.stream(s):
        replay(args.warmup)
    ms_total = timed(replay, args.steps)
    ms_step = ms_total / args.steps
    value = aggregate_gbs(total_bytes, world, ms_step)

    # ---- the same calls launched one by one from Python (launch overhead)
    def stream_calls(nsteps):
        for i in range(nsteps):
            layer(i % ROTATE)

    with torch.cuda.stream(s):
        stream_calls(args.warmup)
    ms_stream = timed(stream_calls, args.steps) / args.steps

    # ---- expert kernel alone (roofline): lists from the routed batch
    logits, probs, _, _ = moe.moe_route(x, Wg, bias, S.k)
    _, _, lists = moe.moe_reselect(logits, probs, S.k, mode, k0, budget)
    torch.cuda.synchronize(dev)
    g_ffn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ffn, stream=s):
        for r in range(ROTATE):
            gg, uu, dd, _ = copies[r]
            moe.moe_expert_ffn(x, gg, uu, dd, lists, S.k, ws, y=y)
    nrep = max(1, args.steps // ROTATE)
    with torch.cuda.stream(s):
        for _ in range(max(1, args.warmup // ROTATE)):
            g_ffn.replay()
    ms_ffn = timed(lambda n: [g_ffn.replay() for _ in range(n)], nrep) / (nrep * ROTATE)
    hbm_peak, peak_kind = measured_peaks()
    ffn_gbs = ffn_bytes / (ms_ffn * 1e-3) / 1e9
    layer_gbs = total_bytes / (ms_step * 1e-3) / 1e9
    if B <= 64:
        # one kernel per call: the fused layer kernel is the dominant kernel,
        # timed by the main region itself
        roofline = {"bound": "hbm", "achieved": layer_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": layer_gbs / hbm_peak, "traffic": NCU_TRAFFIC.get(args.workload),
                    "kernel": "layer_kernel (router, grid barrier, selection, expert stream)",
                    "bytes_per_launch": total_bytes, "us_per_launch": ms_step * 1e3,
                    "peak_source": f"{peak_kind} HBM copy bandwidth",
                    "frac_of_nominal_8tbs": layer_gbs / NOMINAL_HBM_GBS}
    else:
        roofline = {"bound": "hbm", "achieved": ffn_gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": ffn_gbs / hbm_peak, "traffic": NCU_TRAFFIC.get(args.workload),
                    "kernel": "moe_expert_ffn (input prep + grouped SwiGLU expert kernel)",
                    "bytes_per_launch": ffn_bytes, "us_per_launch": ms_ffn * 1e3,
                    "peak_source": f"{peak_kind} HBM copy bandwidth",
                    "frac_of_nominal_8tbs": ffn_gbs / NOMINAL_HBM_GBS}
    expert_leg = {"kernel": "moe_expert_ffn (input prep + expert kernel, lists given)", "achieved": ffn_gbs,
                  "unit": "GB/s", "frac": ffn_gbs / hbm_peak, "us_per_call": ms_ffn * 1e3}

    # ---- the same layers as a stack: the ROTATE weight copies as ROTATE
    # consecutive residual layers, chained on the device (moe_decode_stack)
    xs = torch.zeros(ROTATE + 1, B, S.d, dtype=torch.float32, device=dev)
    xs[0] = x
    stack_layers = [(c[3], bias, c[0], c[1], c[2]) for c in copies]
    stack_ws = moe.new_workspace(B, S.d, S.E, S.k, S.F, dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        moe.moe_decode_stack(xs, stack_layers, S.k, mode, k0, budget, ws=stack_ws, group=group)
    s.synchronize()
    g_stack = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_stack, stream=s):
        moe.moe_decode_stack(xs, stack_layers, S.k, mode, k0, budget, ws=stack_ws, group=group)
    nst = max(1, args.steps // ROTATE)
    with torch.cuda.stream(s):
        for _ in range(max(1, args.warmup // ROTATE)):
            g_stack.replay()
    ms_stack = timed(lambda n: [g_stack.replay() for _ in range(n)], nst) / (nst * ROTATE)
    if moe.moe_check_error(stack_ws, s) != 0:
        raise RuntimeError("device error word set in the stack leg")
    stack = {"layers": ROTATE, "us_per_layer": ms_stack * 1e3,
             "note": "residual stack of the rotating weight copies, layer l+1 chained on layer l"}

    # ---- end to end through the Python API with pinned host buffers
    x_host = torch.from_numpy(x_np).pin_memory()
    y_host = torch.empty(B, S.d, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x)
    y_dev = torch.empty_like(y)

    def e2e_calls(nsteps):
        for i in range(nsteps):
            g, u, dn, wg = copies[i % ROTATE]
            x_dev.copy_(x_host, non_blocking=True)
            moe.moe_layer_decode(x_dev, wg, bias, g, u, dn, S.k, mode, k0, budget, ws=ws, y=y_dev, group=group)
            y_host.copy_(y_dev, non_blocking=True)

    with torch.cuda.stream(s):
        e2e_calls(args.warmup)
    ms_e2e = timed(e2e_calls, args.steps) / args.steps
    e2e = {"value": aggregate_gbs(total_bytes, world, ms_e2e), "unit": UNIT,
           "h2d_bytes_per_step": B * S.d * 4, "d2h_bytes_per_step": B * S.d * 4,
           "ms_per_step": ms_e2e}
    sampler.__exit__(None, None, None)
    clocks = sampler.summary()
    clocks["window"] = "warm-up, timed region, launch-overhead, expert-kernel, stack and end-to-end legs"
    if moe.moe_check_error(ws, s) != 0:
        raise RuntimeError("device error word set during the benchmark")

    extra = {}
    if not args.no_extra and rank == 0 and world == 1:
        extra["host_ms_per_call_python_launch"] = ms_stream
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "B": B, "d": S.d, "E": S.E, "k": S.k, "d_ff": S.F,
                   "rule": w["rule"], "n_active": n_active, "bytes_per_call": total_bytes,
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {ROTATE} rotating copies of the layer weights "
                         f"({3 * S.E * S.d * S.F * 2 / 1e9:.2f} GB of experts + the router each)",
                   "launch": ("CUDA graph of 4 layer calls, one cooperative kernel per call" if B <= 64 else
                              "CUDA graph of 4 layer calls, 4 kernels per call chained with PDL")},
        "us_per_call": ms_step * 1e3,
        "frac_of_nominal_8tbs": (total_bytes / (ms_step * 1e-3) / 1e9) / NOMINAL_HBM_GBS,
        "frac_of_measured_hbm": (total_bytes / (ms_step * 1e-3) / 1e9) / hbm_peak,
        "stream_launch_us_per_call": ms_stream * 1e3,
        "roofline": roofline,
        "expert_ffn_leg": expert_leg,
        "stack_leg": stack,
        "e2e": e2e,
        # up to 64 tokens one fused kernel per call; above, router,
        # selection, x dispatch and expert kernels
        "gpu_launches": (1 if B <= 64 else 4) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, S, L, x_np)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_all, g_one, g_ffn, g_stack
    torch.cuda.synchronize(dev)


SWEEP = {
    # shape: [(B, mode, k0, budget, token kind[, tokens per request])], the
    # configurations the results table reports (one weight set per shape,
    # ROTATE copies); mode 4 (hierarchical XShare) takes the request size
    "tiny": [(4, 1, 2, 0, "normal"), (4, 0, 0, 0, "normal")],
    "e64": [(16, 1, 4, 0, "normal"), (16, 0, 0, 0, "normal")],
    "q30b": [(b, m, k0, 0, "normal") for b in (1, 4, 8, 16, 32, 48, 64, 128) for (m, k0) in ((0, 0), (1, 4))]
            + [(16, 1, k0, 0, "normal") for k0 in (2, 6, 8)]
            + [(32, 0, 0, 0, "spec")] + [(32, 2, 0, m, "spec") for m in (24, 32, 48)]
            + [(16, 3, 0, 0, "normal"), (64, 3, 0, 0, "normal"), (32, 3, 0, 0, "spec")]
            + [(32, 4, 0, m, "spec", 4) for m in (24, 32, 48)],
    "q235b": [(b, 1, 4, 0, "normal") for b in (1, 8, 16, 64)] + [(16, 0, 0, 0, "normal")],
}


def channel_bytes(keep_bits: np.ndarray, sel: np.ndarray, d: int, F: int, B: int, k: int) -> int:
    """Algorithmic bytes of one channel top-k call: for every activated
    expert, the union of its pairs' kept channels, each a gate row, an up row
    and a channel-major down row of 2 d bytes (whole 32-byte sectors, since
    2 d is a multiple of 128); plus the scores, x and y."""
    bits = np.unpackbits(keep_bits.view(np.uint8), bitorder="little").reshape(B, k, F)
    weights = 0
    for e in np.unique(sel[sel >= 0]):
        u = np.zeros(F, bool)
        for b, slot in zip(*np.nonzero(sel == e)):
            u |= bits[b, slot].astype(bool)
        weights += int(u.sum()) * 3 * 2 * d
    return weights + B * k * F * 4 + 2 * B * d * 4


def run_channels(args, w, rank, world, local_rank):
    """Per-token channel top-k inside the activated experts: routing and
    selection as for the layer (moe_route, moe_reselect), then
    moe_expert_ffn_channels timed alone over graph replays on ROTATE weight
    copies (each with its channel-major down copy)."""
    import torch
    import aware_expert_routing_moe_b200 as moe
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    S = ms.SHAPES[w["shape"]]
    B = w["B"]
    c = max(1, int(round(w["channels"] * S.F)))
    L = ms.make_weights(S, 0)
    x_np = ms.make_tokens(S, B, 0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    x, Wg, bias = t(x_np), t(L["Wg"]), t(L["bias"])
    base = (t(L["Wgate"].view(np.int16)), t(L["Wup"].view(np.int16)), t(L["Wdown"].view(np.int16)))
    copies = [base] + [tuple(a.clone() for a in base) for _ in range(ROTATE - 1)]
    downT = [moe.moe_down_channel_major(cp[2]) for cp in copies]
    logits, probs, _, _ = moe.moe_route(x, Wg, bias, S.k)
    sel, sw, _ = moe.moe_reselect(logits, probs, S.k, w["mode"], w["k0"], w["budget"])
    score = t(np.random.default_rng(1000).standard_normal((B, S.k, S.F)).astype(np.float32))
    y = torch.empty(B, S.d, dtype=torch.float32, device=dev)
    keep = torch.empty(B, S.k, S.F // 32, dtype=torch.int32, device=dev)
    ws = torch.zeros(moe.load_library().moe_channels_workspace_bytes(moe.Dims(B, S.d, S.E, S.k, S.F)),
                     dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))

    def call(r):
        g, u, _ = copies[r]
        moe.moe_expert_ffn_channels(x, g, u, downT[r], sel, sw, score, c, y=y, keep=keep, ws=ws)

    with torch.cuda.stream(s):
        for r in range(ROTATE):
            call(r)
    s.synchronize()
    nbytes = channel_bytes(keep.cpu().numpy(), sel.cpu().numpy(), S.d, S.F, B, S.k)
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all, stream=s):
        for r in range(ROTATE):
            call(r)
    reps = max(1, args.steps // ROTATE)
    with torch.cuda.stream(s):
        for _ in range(max(1, args.warmup // ROTATE)):
            g_all.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    with sampler, torch.cuda.stream(s):
        e0.record(s)
        for _ in range(reps):
            g_all.replay()
        e1.record(s)
        e1.synchronize()
    ms_call = e0.elapsed_time(e1) / (reps * ROTATE)
    if moe.moe_check_error(ws, s) != 0:
        raise RuntimeError("device error word set in the channel path")
    hbm_peak, peak_kind = measured_peaks()
    gbs = nbytes / (ms_call * 1e-3) / 1e9
    line = {
        "metric": "per-token channel top-k expert FFN: µs and achieved HBM GB/s of the sector-counted bytes",
        "value": gbs, "unit": UNIT, "n_gpus": 1, "steps": reps * ROTATE, "warmup": args.warmup,
        "ms_per_step": ms_call, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w), "channels_kept": c, "bytes_per_call": nbytes,
                   "l2": f"{ROTATE} rotating copies of the expert weights"},
        "us_per_call": ms_call * 1e3,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                     "traffic": NCU_TRAFFIC.get(args.workload),
                     "kernel": "channel_select + channel_items + channel_stream kernels (traffic: channel_stream)",
                     "peak_source": f"{peak_kind} HBM copy bandwidth"},
        "gpu_launches": 3 * reps * ROTATE, "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    del g_all


def run_sweep(args):
    """Times moe_layer_decode on every configuration of SWEEP (device time per
    call over graph replays of ROTATE calls on rotating weight copies) and
    the oracle on one call (1 thread and all host threads); one JSON line
    per configuration."""
    import torch
    import aware_expert_routing_moe_b200 as moe
    import oracle
    dev = torch.device("cuda", 0)
    moe.load_library()
    cores = len(os.sched_getaffinity(0))
    hbm_peak, _ = measured_peaks()
    shapes = args.sweep.split(",") if args.sweep != "all" else list(SWEEP)
    for shape in shapes:
        S = ms.SHAPES[shape]
        L = ms.make_weights(S, 0)
        t = lambda a: torch.from_numpy(a).to(dev)
        base = (t(L["Wgate"].view(np.int16)), t(L["Wup"].view(np.int16)), t(L["Wdown"].view(np.int16)), t(L["Wg"]))
        copies = [base] + [tuple(c.clone() for c in base) for _ in range(ROTATE - 1)]
        bias = t(L["bias"])
        s = torch.cuda.Stream(dev)
        for row in SWEEP[shape]:
            B, mode, k0, budget, kind = row[:5]
            group = row[5] if len(row) > 5 else 1
            x_np = ms.make_tokens(S, B, 0, kind=kind)
            x = t(x_np)
            ws = moe.new_workspace(B, S.d, S.E, S.k, S.F, dev)
            y = torch.empty(B, S.d, dtype=torch.float32, device=dev)
            nact_t = torch.zeros(4, dtype=torch.int32, device=dev)
            s.wait_stream(torch.cuda.current_stream(dev))

            def layer(r):
                g, u, dn, wg = copies[r]
                moe.moe_layer_decode(x, wg, bias, g, u, dn, S.k, mode, k0, budget, ws=ws, y=y, n_active=nact_t,
                                     group=group)

            with torch.cuda.stream(s):
                for r in range(ROTATE):
                    layer(r)
            s.synchronize()
            g_all = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_all, stream=s):
                for r in range(ROTATE):
                    layer(r)
            with torch.cuda.stream(s):
                for _ in range(5):
                    g_all.replay()
            torch.cuda.synchronize(dev)
            reps = max(args.steps // ROTATE, 5)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s):
                e0.record(s)
                for _ in range(reps):
                    g_all.replay()
                e1.record(s)
            e1.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / (reps * ROTATE)
            if moe.moe_check_error(ws, s) != 0:
                raise RuntimeError(f"device error word set: {shape} {B} {mode}")
            n_active = int(nact_t[0].item())
            total, _ = algorithmic_bytes(S, B, n_active)
            gbs = total / (us * 1e-6) / 1e9
            line = {"shape": shape, "B": B, "mode": ["NONE", "OEA", "XShare", "Affinity", "XShareHier"][mode],
                    "k0": k0, "budget": budget, "group": group, "tokens": kind, "n_active": n_active, "us": us,
                    "bytes": total, "GBps": gbs, "frac_8tbs": gbs / NOMINAL_HBM_GBS,
                    "frac_measured": gbs / hbm_peak}
            if not args.no_cpu_baseline:
                ms_t = []
                for th in (1, cores):
                    t0 = time.perf_counter()
                    oracle.layer(x_np, L, S.k, mode, k0, budget, threads=th, group=group)
                    ms_t.append((time.perf_counter() - t0) * 1e3)
                line["oracle_ms_1"] = ms_t[0]
                line["oracle_ms_n"] = ms_t[1]
                line["oracle_cores"] = cores
            print(json.dumps(line), flush=True)
            del g_all
        del copies, base
        torch.cuda.empty_cache()
    return 0


def run_profile_case(args, w):
    """A small case for ncu captures: one weight copy (about 1.2 GB for the
    Qwen3-30B shape, so the activated experts still exceed L2), `warmup`
    layer calls, then `steps` more, launched from the stream, no timing.
    Channel workloads: routing and selection once, then the channel top-k
    calls; the sector-counted bytes of one call are printed."""
    import torch
    import aware_expert_routing_moe_b200 as moe
    S = ms.SHAPES[w["shape"]]
    B = w["B"]
    L = ms.make_weights(S, 0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    x = t(ms.make_tokens(S, B, 0, kind=w.get("kind", "normal")))
    Wg, bias = t(L["Wg"]), t(L["bias"])
    g, u, dn = (t(L[n].view(np.int16)) for n in ("Wgate", "Wup", "Wdown"))
    if "channels" in w:
        c = max(1, int(round(w["channels"] * S.F)))
        downT = moe.moe_down_channel_major(dn)
        logits, probs, _, _ = moe.moe_route(x, Wg, bias, S.k)
        sel, sw, _ = moe.moe_reselect(logits, probs, S.k, w["mode"], w["k0"], w["budget"])
        score = t(np.random.default_rng(1000).standard_normal((B, S.k, S.F)).astype(np.float32))
        keep = torch.empty(B, S.k, S.F // 32, dtype=torch.int32, device="cuda")
        cws = torch.zeros(moe.load_library().moe_channels_workspace_bytes(moe.Dims(B, S.d, S.E, S.k, S.F)),
                          dtype=torch.uint8, device="cuda")
        for _ in range(args.warmup + args.steps):
            moe.moe_expert_ffn_channels(x, g, u, downT, sel, sw, score, c, keep=keep, ws=cws)
        torch.cuda.synchronize()
        status = moe.moe_check_error(cws)
        nbytes = channel_bytes(keep.cpu().numpy(), sel.cpu().numpy(), S.d, S.F, B, S.k)
        print(f"profile case {args.workload}: {args.warmup}+{args.steps} channel calls, status {status}, "
              f"sector-counted bytes per call {nbytes}")
        return 0 if status == 0 else 1
    ws = moe.new_workspace(B, S.d, S.E, S.k, S.F)
    for _ in range(args.warmup + args.steps):
        moe.moe_layer_decode(x, Wg, bias, g, u, dn, S.k, w["mode"], w["k0"], w["budget"], ws=ws,
                             group=w.get("group", 1))
    torch.cuda.synchronize()
    status = moe.moe_check_error(ws)
    print(f"profile case {args.workload}: {args.warmup}+{args.steps} layer calls, status {status}")
    return 0 if status == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="q30b_b16_oea4")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", default=None,
                    help="time every results-table configuration of these shapes ('all' or a comma list)")
    ap.add_argument("--profile", action="store_true",
                    help="small case for ncu: one weight copy, warmup + steps layer calls, no timing")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = WORKLOADS[args.workload]
    if args.sweep:
        return run_sweep(args)
    if args.profile:
        return run_profile_case(args, w)
    if "channels" in w and args.impl == "ours":
        if rank == 0:
            run_channels(args, w, rank, world, local_rank)
        return 0
    if args.impl == "reference":
        run_reference(args, w, rank)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
