#!/usr/bin/env python
"""Decode benchmark of the predictor-gated sparse FFN stack.

One step = one decode token through the whole stack (every layer: rmsnorm,
predictor, compaction, gathered up/gate + activation, gathered split-K down
projection, residual) of the Llama2-70B-shaped ReGLU Q4_0 workload (80
layers, d_model 8192, d_ff 28672, batch 1) on seeded synthetic weights
generated in place on the GPU.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pi|reference]

N > 1 runs under torch.distributed.run, one process per GPU; every rank
decodes its own token stream through its own copy of the stack (the decode
step has no data-path exchange), so scaling is weak and `value` sums the
ranks' tokens over the slowest rank's time.

--impl reference times the CPU oracle on the host cores instead: the same
workload and metric, each step one token through a bounded sample of the
layers, extrapolated to the whole stack.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-FFN decode tokens/s (Llama2-70B Q4_0 shape)"


def metric_name(workload: str, batch: int) -> str:
    """The headline metric for the headline workload at batch 1, else a
    name that says which workload and batch the line measures."""
    if workload == DEFAULT_WORKLOAD and batch == 1:
        return METRIC
    return f"sparse-FFN tokens/s ({workload}, batch {batch})"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "llama2_70b_reglu_8192x28672_q4_0"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="pi", choices=["pi", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--mode", default="per_token", choices=["per_token", "union"])
    ap.add_argument("--cpu-sample-layers", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the first N layers (profiling captures; 0 = all)")
    ap.add_argument("--cold-tier", default="none", choices=["none", "host"],
                    help="host: every layer's cold rows (neurons >= hot) in page-locked host "
                         "memory, read by the GPU over the host link")
    return ap.parse_args()


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while
    the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev: int, interval=0.02):
        self.samples, self.reasons, self.ok = [], set(), False
        self.interval = interval
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            p = torch.cuda.get_device_properties(torch_dev)
            try:
                bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report it, keep running
            self.err = repr(e)

    def _sample(self):
        nv = self.nv
        mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append(mhz)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "note": getattr(self, "err", "no samples")}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "pi" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        # a short limit: a rank that waits for one that died ends with an error
        limit = float(os.environ.get("PI_DIST_TIMEOUT_S", "180"))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=limit))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ accounting

def weight_row_bytes(dtype: str, d: int) -> float:
    return {"f32": 4.0 * d, "f16": 2.0 * d, "q4_0": d / 2 + (d // 32) * 2}[dtype]


def predictor_bytes(w) -> float:
    pb = {"f32": 4.0, "f16": 2.0}[w.p_dtype]
    return (w.rank * w.d_model + (w.d_ff - w.hot) * w.rank) * pb + (w.d_ff - w.hot) * 4


def layer_algorithmic_bytes(w, rows_listed: int, rows_down: int, n_layers: int,
                            rows_second: int | None = None) -> dict:
    """Algorithmic bytes of each kernel kind summed over a run in which the
    FFN launches read `rows_listed` first-matrix rows (W_gate for ReGLU,
    W_up otherwise), `rows_second` W_up rows (ReGLU; None = one per listed
    row, as the batch kernels read them) and `rows_down` w_down_t rows, over
    `n_layers` layer evaluations (batch 1)."""
    rb = weight_row_bytes(w.w_dtype, w.d_model)
    d4 = 4.0 * w.d_model
    words = (w.d_ff + 31) // 32
    if rows_second is None:
        rows_second = rows_listed if w.act == "reglu" else 0
    return {
        "rmsnorm": n_layers * 2 * d4,
        "pred_u": n_layers * (w.rank * w.d_model * {"f32": 4, "f16": 2}[w.p_dtype] + d4 + 4 * w.rank),
        "pred_z": n_layers * ((w.d_ff - w.hot) * w.rank * {"f32": 4, "f16": 2}[w.p_dtype]
                              + (w.d_ff - w.hot) * 4 + 4 * w.rank + 4 * words),
        "compact": n_layers * 4.0 * words,
        "ffn_up": rows_listed * (rb + 4 + 4) + rows_second * rb + n_layers * (d4 + 4 * words),
        "ffn_down": rows_down * rb,
        "reduce": 0.0,  # partials live in L2; counted as traffic only by ncu
    }


# ---------------------------------------------------------------- CPU leg

def cpu_oracle_tokens_per_s(w, n_sample_layers: int, reps: int, step0: int = 0):
    """Times the CPU oracle (as it stands) on one token through
    `n_sample_layers` layers `reps` times; returns (tokens/s extrapolated to
    the whole stack, threads used, seconds per layer, description)."""
    from activation_sparse_predictor_b200 import synth
    from oracle import Oracle
    orc = Oracle()
    layers = [synth.layer_host(w, l) for l in range(n_sample_layers)]
    x = synth.x_host(w, step0, 1)[0]
    per_layer = []
    for r in range(reps):
        xr = x.copy()
        for L in layers:
            t0 = time.perf_counter()
            xo, _, _ = orc.layer_forward(L, xr, w.tau)
            per_layer.append(time.perf_counter() - t0)
            xr = xo.astype("float32")
    s = statistics.median(per_layer)
    tps = 1.0 / (s * w.n_layers)
    desc = (f"oracle (plain C, double accumulation, OpenMP) on one token through "
            f"{n_sample_layers} of {w.n_layers} layers x {reps}; median seconds per layer "
            f"{s:.3f} extrapolated to the {w.n_layers}-layer stack")
    return tps, orc.num_threads(), s, desc


def cpu_oracle_variants(w, budget_s: float = 12.0) -> dict:
    """The oracle as it stands, on one token through one layer of the
    workload, timed four ways: the sparse layer (predictor, compaction, FFN
    over the predicted set: the method) and the dense FFN (every neuron), each
    on all host threads and on one thread.  Repetitions stop once a variant
    has used its share of `budget_s`.  Returns {variant: {...}}."""
    from activation_sparse_predictor_b200 import synth
    from oracle import Oracle
    orc = Oracle()
    all_threads = orc.num_threads()
    L = synth.layer_host(w, 0)
    x = synth.x_host(w, 0, 1)[0]
    xh = orc.rmsnorm(x)

    def sparse():
        orc.layer_forward(L, x, w.tau)

    def dense():
        orc.dense_ffn(L, xh)

    out = {}
    share = budget_s / 4.0
    try:
        for name, fn in (("sparse", sparse), ("dense", dense)):
            for threads in (all_threads, 1):
                orc.set_num_threads(threads)
                times = []
                t_start = time.perf_counter()
                while not times or (time.perf_counter() - t_start < share and len(times) < 5):
                    t0 = time.perf_counter()
                    fn()
                    times.append(time.perf_counter() - t0)
                s = statistics.median(times)
                key = f"{name}_{'all_threads' if threads == all_threads else '1_thread'}"
                out[key] = {"tokens_per_s": 1.0 / (s * w.n_layers), "seconds_per_layer": s,
                            "threads": threads, "reps": len(times)}
    finally:
        orc.set_num_threads(all_threads)
    return out


def run_reference(args, world, rank):
    """CPU oracle arm: rank 0 only, bounded sample per step."""
    if rank != 0:
        return
    if args.batch != 1:
        print(json.dumps({"impl": "reference",
                          "unavailable": "the oracle arm times single-token decode (batch 1) only"}),
              flush=True)
        return
    from activation_sparse_predictor_b200 import build, synth
    build.build_synth()
    w = synth.WORKLOADS[args.workload]
    from oracle import Oracle
    from oracle.build import build as build_oracle
    build_oracle()
    orc = Oracle()
    n_sample = min(args.cpu_sample_layers, w.n_layers)
    layers = [synth.layer_host(w, l) for l in range(n_sample)]
    per_step = []
    for step in range(args.warmup + args.steps):
        x = synth.x_host(w, step, 1)[0]
        t0 = time.perf_counter()
        for L in layers:
            xo, _, _ = orc.layer_forward(L, x, w.tau)
            x = xo.astype("float32")
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            per_step.append(dt)
    sec_per_layer = sum(per_step) / (len(per_step) * len(layers))
    tps = 1.0 / (sec_per_layer * w.n_layers)
    sample = (f"each step: one token through {len(layers)} of {w.n_layers} layers "
              f"(host-generated, resident); tokens/s extrapolated to all {w.n_layers} layers")
    line = {
        "impl": "reference", "metric": metric_name(w.name, 1), "value": tps, "unit": UNIT,
        "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * sec_per_layer * w.n_layers,
        "ms_per_step_basis": (f"extrapolated: measured {1000.0 * sec_per_layer:.1f} ms per layer "
                              f"over {len(layers)} sampled layers x {args.steps} steps, times "
                              f"{w.n_layers} layers"),
        "ms_per_sampled_step": 1000.0 * sum(per_step) / len(per_step),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generator; no weights or datasets)",
        "config": run_config(w, args.batch, args.mode, w.n_layers, args.gpus,
                             l2_mode_for(w, w.n_layers, B200_L2_BYTES)),
        "cpu_baseline": {"value": tps, "unit": UNIT, "cores": orc.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tps, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PROFILES = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles")
CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "activation_sparse_predictor_b200", "csrc")


FUSED_SOURCES = ("pi_stack.cu", "pi_stack.cuh", "pi_common.cuh")


def kernel_source_sha256() -> str:
    """Hash of the sources the fused single-token kernel is built from."""
    h = hashlib.sha256()
    for name in FUSED_SOURCES:
        h.update(name.encode())
        h.update(open(os.path.join(CSRC, name), "rb").read())
    return h.hexdigest()


def measured_traffic_per_layer(workload: str):
    """DRAM bytes (read + write) per layer of the fused kernel from the
    committed ncu summary of this workload, or None when there is none or it
    was taken on other kernel sources than the ones built now."""
    path = os.path.join(PROFILES, f"fused_stack_{workload}_ncu.md")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        m = re.match(r"^- (source_sha256|dram_bytes_per_layer): `?([0-9a-fA-Fe.+]+)`?\s*$", line.strip())
        if m:
            vals[m.group(1)] = m.group(2)
    if vals.get("source_sha256") != kernel_source_sha256() or "dram_bytes_per_layer" not in vals:
        return None
    return float(vals["dram_bytes_per_layer"])


def workload_config(w, batch, mode, l2="streamed"):
    l2_text = {
        "streamed": "inputs larger than L2: every step streams the whole stack's weights "
                    "and predictors from HBM (no flush needed)",
        "flushed": "weights fit in L2: a 2 x L2 buffer is written between timed steps, each "
                   "step timed on its own (cold L2)",
        "resident": "weights fit in L2 and stay resident across back-to-back steps "
                    "(L2-resident figure)",
    }[l2]
    return {"workload": w.name, "layers": w.n_layers, "d_model": w.d_model, "d_ff": w.d_ff,
            "hot_prefix": w.hot, "predictor_rank": w.rank, "activation": w.act,
            "weights": w.w_dtype, "predictor_weights": w.p_dtype, "batch": batch,
            "mask_mode": mode, "tau": w.tau, "l2": l2_text}


B200_L2_BYTES = 126 * 2 ** 20  # used where no device is at hand (the CPU arm)


def l2_mode_for(w, n_layers: int, l2_bytes: int) -> str:
    """'flushed' when the stack's weights would fit twice in L2 (then each
    step is timed on its own after a 2 x L2 write), else 'streamed'."""
    from activation_sparse_predictor_b200 import synth
    return "flushed" if n_layers * synth.layer_nbytes(w) < 2 * l2_bytes else "streamed"


def run_config(w, batch, mode, n_layers, world, l2="streamed", cold_tier="none"):
    """The `config` object both arms print for a run (same keys)."""
    c = dict(workload_config(w, batch, mode, l2), layers=n_layers,
             parallelism=f"replicas x{world}" if world > 1 else "single GPU")
    if cold_tier == "host":
        c["cold_tier"] = "rows of neurons >= hot in page-locked host memory"
    return c


def host_link_peak(dev, stream) -> float:
    """GB/s of a 1 GiB copy from page-locked host memory to the device (the
    best of 3), the bound for rows read from a host-memory cold tier."""
    import torch
    n = 1 << 30
    h = torch.empty(n, dtype=torch.uint8).pin_memory()
    d = torch.empty(n, dtype=torch.uint8, device=dev)
    best = 0.0
    with torch.cuda.stream(stream):
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            d.copy_(h, non_blocking=True)
            b.record(stream)
            b.synchronize()
            best = max(best, n / (a.elapsed_time(b) / 1000.0) / 1e9)
    del h, d
    return best


# ---------------------------------------------------------------- GPU leg

def run_pi(args, world, rank, local):
    import torch

    from activation_sparse_predictor_b200 import pi, synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    B = args.batch
    mode = pi.MODES[args.mode]
    nl = args.layers if 0 < args.layers < w.n_layers else w.n_layers
    layers = []
    for l in range(nl):
        t = synth.layer_device(w, l, dev)
        layers.append(pi.Layer.packed(
            w, {k: t[k] for k in ("w_gate", "w_up", "w_down_t", "bias", "p1", "p2", "p_bias")
                if k in t}))
        del t
    if args.cold_tier == "host":
        layers = [L.with_host_cold_tier() for L in layers]
    arr = pi.layer_array(layers)
    K, W = args.steps, max(3, args.warmup)
    xs = torch.stack([synth.x_device(w, rank * 1_000_003 + s, B, dev) for s in range(K + W)])
    stream = torch.cuda.Stream(dev)
    ws = pi.workspace(layers, B, dev, stream)
    x = torch.empty((B, w.d_model), dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    with torch.cuda.stream(stream):
        # eager warm-up: also settles shared-memory attributes before capture
        for i in range(2):
            x.copy_(xs[i])
            pi.pi_ffn_stack(layers, x, w.tau, mode, ws=ws, stream=stream, _arr=arr)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        n_before = pi.pi_kernel_launches()
        # (relaxed: the cold tier's host pointers are looked up at the call)
        with torch.cuda.graph(g, stream=stream,
                              capture_error_mode="relaxed" if args.cold_tier == "host" else "global"):
            pi.pi_ffn_stack(layers, x, w.tau, mode, ws=ws, stream=stream, _arr=arr)
        kernels_per_step = pi.pi_kernel_launches() - n_before  # what one replay launches
        for i in range(W):
            x.copy_(xs[i])
            g.replay()
    stream.synchronize()
    st, word = pi.pi_get_device_status(ws, stream=stream)
    assert st == pi.PI_OK, f"device status {word:#x} after warm-up"
    pi.pi_read_counters(ws, clear=True, stream=stream)
    pi.pi_read_cold_counters(ws, clear=True, stream=stream)

    # ---- timed region: K graph replays, inputs already in HBM.  A stack
    # whose weights fit in L2 is timed step by step with a 2 x L2 write
    # between steps (cold L2); larger stacks stream from HBM on every step.
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    l2_mode = l2_mode_for(w, nl, l2_bytes)
    flush = (torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev)
             if l2_mode == "flushed" else None)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)] if flush is not None else []
    sampler = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for i in range(K):
                x.copy_(xs[W + i])
                if flush is not None:
                    flush.fill_(float(i))
                    step_ev[i][0].record(stream)
                g.replay()
                if flush is not None:
                    step_ev[i][1].record(stream)
            ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    ms = ev0.elapsed_time(ev1) if flush is None else sum(a.elapsed_time(b) for a, b in step_ev)
    rows_listed, rows_down, rows_second = pi.pi_read_counters(ws, clear=True, stream=stream)
    cold_rows = pi.pi_read_cold_counters(ws, clear=True, stream=stream)
    ms_max = max_over_ranks(ms, world, dev)
    value = world * K * B / (ms_max / 1000.0)
    resident = None
    if flush is not None:
        # the same steps back to back, weights left in L2 (reported beside the number)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            r0.record(stream)
            for i in range(K):
                x.copy_(xs[W + i])
                g.replay()
            r1.record(stream)
        torch.cuda.synchronize(dev)
        pi.pi_read_counters(ws, clear=True, stream=stream)
        resident = K * B / (r0.elapsed_time(r1) / 1000.0)

    # ---- per-kernel device times: one profiled pass over the same step inputs
    x.copy_(xs[W])
    pi.pi_read_counters(ws, clear=True, stream=stream)
    prof = pi.pi_ffn_stack_profile(layers, x, w.tau, mode, ws=ws, stream=stream, _arr=arr)
    pr_listed, pr_down, pr_second = pi.pi_read_counters(ws, clear=True, stream=stream)
    prof = {k: v for k, v in prof.items() if v[1] > 0}
    # the persistent kernel alone at several tokens (Q4_0 stacks with
    # per-token masks) makes one pass over the stack per token, so the
    # predictor and the per-layer vectors are read once per layer and token
    passes = B if (B > 1 and set(prof) == {"fused_stack"}) else 1

    # bytes actually read per step (predictor + listed rows + nonzero down rows)
    by = layer_algorithmic_bytes(w, rows_listed, rows_down, K * nl * passes, rows_second)
    step_bytes = sum(by.values()) / K
    peak, peak_kind = hbm_peak()
    step_gbs = step_bytes / (ms / K / 1000.0) / 1e9
    pby = layer_algorithmic_bytes(w, pr_listed, pr_down, nl * passes, pr_second)
    pby["fused_stack"] = sum(pby.values())  # the fused kernel runs every step
    dom = max(prof, key=lambda k: prof[k][0])
    dom_ms, dom_n = prof[dom]
    if len(prof) == 1:
        # one kernel kind makes the whole step: take its launch time from the
        # timed graph replays that give `value`, and its bytes from their counters
        timing_source = "graph replays of the timed region (the same timing as value)"
        dom_ms = ms / K * dom_n / prof[dom][1]
        dom_bytes_per_launch = step_bytes / dom_n
    else:
        timing_source = "profiled eager pass with CUDA events around every launch"
        dom_bytes_per_launch = pby[dom] / dom_n
    achieved = dom_bytes_per_launch / (dom_ms / dom_n / 1000.0) / 1e9
    # DRAM traffic per launch from the committed ncu capture of this kernel
    # (per layer, scaled to the layers of an average launch); null when the
    # capture was taken on other kernel sources
    tpl = measured_traffic_per_layer(w.name) if dom == "fused_stack" else None
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_kind,
                "traffic": tpl * nl * passes / dom_n if tpl is not None else None,
                "algorithmic_bytes_per_launch": dom_bytes_per_launch,
                "avg_launch_us": 1000.0 * dom_ms / dom_n, "timing_source": timing_source,
                "per_kind_ms_per_step": {k: v[0] for k, v in prof.items()},
                "launches_per_step": {k: v[1] for k, v in prof.items()}}
    if args.cold_tier == "host":
        # the rows read from host memory bound the step: bytes that crossed
        # the host link per step over the step time, against a pinned copy
        cold_bytes = sum(cold_rows) * weight_row_bytes(w.w_dtype, w.d_model) / K
        link = host_link_peak(dev, stream)
        achieved = cold_bytes / (ms / K / 1000.0) / 1e9
        roofline = {"bound": "host_link", "kernel": "ffn_up + ffn_down (rows >= hot)",
                    "achieved": achieved, "peak": link, "unit": "GB/s", "frac": achieved / link,
                    "peak_source": "page-locked host-to-device copy of 1 GiB, measured in this run",
                    "traffic": None, "host_bytes_per_step": cold_bytes,
                    "host_rows_per_step": {"first_read": cold_rows[0] / K,
                                           "down_read": cold_rows[1] / K,
                                           "second_read": cold_rows[2] / K},
                    "device_bytes_per_step": step_bytes - cold_bytes,
                    "timing_source": "graph replays of the timed region (the same timing as value)",
                    "per_kind_ms_per_step": {k: v[0] for k, v in prof.items()},
                    "launches_per_step": {k: v[1] for k, v in prof.items()}}

    # ---- end to end through the C ABI with host buffers: pinned H2D of the
    # step's input, the stack, D2H of the step's output, every step
    hx = torch.empty((K, B, w.d_model), dtype=torch.float32).pin_memory()
    hx.copy_(xs[W:W + K].cpu())
    hy = torch.empty((K, B, w.d_model), dtype=torch.float32).pin_memory()
    barrier(world)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K):
            x.copy_(hx[i], non_blocking=True)
            g.replay()
            hy[i].copy_(x, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = {"value": world * K * B / (e2e_ms / 1000.0), "unit": UNIT,
           "h2d_bytes_per_step": B * w.d_model * 4, "d2h_bytes_per_step": B * w.d_model * 4}
    assert bool(torch.isfinite(hy).all())

    st, word = pi.pi_get_device_status(ws, stream=stream)
    assert st == pi.PI_OK, f"device status {word:#x}"
    del g
    if rank != 0:
        return

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        # ~10 s of oracle work: the sample layers, 24 passes (the sparse layer
        # on every host thread: the reported value), then the sparse and the
        # dense layer on one thread and on all threads (~12 s)
        tps, cores, s, desc = cpu_oracle_tokens_per_s(w, args.cpu_sample_layers, 24)
        cpu = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "variants": cpu_oracle_variants(w)}

    line = {
        "metric": metric_name(w.name, B), "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded generator, weights generated on the GPU; no datasets)",
        "config": run_config(w, B, args.mode, nl, world, l2_mode, args.cold_tier),
        "hbm_gbs_actual": step_gbs, "hbm_frac_of_peak": step_gbs / peak,
        "bytes_per_step": step_bytes,
        "rows_per_step": {"first_read": rows_listed / K, "second_read": rows_second / K,
                          "down_read": rows_down / K},
        "l2_resident_value": resident,
        "clocks": sampler.summary(),
        "e2e": e2e,
        "gpu_launches": K * kernels_per_step,
        "roofline": roofline,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_pi(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
