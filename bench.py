#!/usr/bin/env python
"""Benchmark of the FP8 x FP4 MoE layer forward on B200.

One step = moe_plan + moe_forward (permute -> linear1 + SwiGLU + requant ->
linear2 x top-k weight -> combine) over one batch of the workload, inputs
resident in HBM, L2 flushed (256 MB write) before every timed step.  Times
are CUDA events on the launching stream.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

Default: the headline is the largest config, the usage-example layer (T=8192,
H=7168, I=9216, E=8, top-2); every other config (mid, skewed, decode at
T=128/64/32/16) is measured the same way at N = 1 and reported under
"configs" in the same line.  --workload NAME times NAME alone.

Multi-GPU: replicas (each rank runs its own batch of the workload with its
own activations; no collective on the data path); the step time is the max
over ranks and `value` counts the work of every rank ("scaling": "weak").
`--impl reference` times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload, on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd TFLOPS & tokens/s on 1 B200; % of tensor/HBM roofline"

# DRAM traffic (read + write bytes) of one linear1 launch on the usage workload (full size)
# from one ncu capture (summarised, with its command, under profiles/).  Reported only while
# the kernel sources still hash to the value they had when the counters were taken;
# otherwise the traffic is unknown (null).
LINEAR1_TRAFFIC = {"workload": "usage", "bytes": 1241.526016e6 + 152.760576e6,
                   "sources_sha256_16": "6b76f8d1d804e3d8"}
LINEAR1_SOURCES = ["moe_gemm.cu", "moe_epilogue.cuh", "moe_device.cuh", "sm100_ptx.cuh",
                   "moe_internal.cuh"]


def _linear1_traffic(workload_name):
    import hashlib
    h = hashlib.sha256()
    for f in LINEAR1_SOURCES:
        with open(os.path.join(ROOT, "block_scaled_fp8_permute_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if (workload_name == LINEAR1_TRAFFIC["workload"]
            and h.hexdigest()[:16] == LINEAR1_TRAFFIC["sources_sha256_16"]):
        return LINEAR1_TRAFFIC["bytes"]
    return None
L2_FLUSH_BYTES = 256 << 20


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=None,
                   help="time only this workload (default: the usage config as the headline "
                        "plus every other config as a sub-record)")
    p.add_argument("--no-sub", action="store_true", help="headline only, no sub-records")
    p.add_argument("--sub-cpu-seconds", type=float, default=4.0,
                   help="target CPU time of each sub-record's oracle sample")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--gemm-variant", type=int, default=None,
                   help="moe_set_gemm_variant before timing (0 one-SM tiles, 1 SM pairs)")
    p.add_argument("--swap-max", type=int, default=None, help="moe_set_swap_max before timing")
    p.add_argument("--narrow", type=int, default=None,
                   help="moe_set_narrow_tiles before timing (-1 auto, 0 off, 1 on)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the bounded oracle sample")
    return p.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, src="fallback")


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every ~0.2 ms in a
    background thread.  mark("start") / mark("end") bracket the timed region;
    the sampler may keep running over later steps of the same workload, which
    summary() reports separately."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples, self.max_mhz, self.err, self.marks = [], None, None, {}

    def _handle(self, nv):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            return nv.nvmlDeviceGetHandleByUUID(uuid.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def mark(self, name):
        self.marks[name] = time.perf_counter()

    def wait_first(self, timeout=1.0):
        """Block until the sampling thread has taken its first sample (its start-up
        and NVML's first call would otherwise eat a short timed region)."""
        t_end = time.perf_counter() + timeout
        while self.nv is not None and not self.samples and time.perf_counter() < t_end:
            time.sleep(0.0005)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv, self.h = nv, self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report it instead of clocks
            self.err, self.nv = f"nvml unavailable: {e}", None
            return self
        self.stop = threading.Event()

        def loop():
            while not self.stop.is_set():
                try:
                    mhz = float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((time.perf_counter(), mhz, bits))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.0002)

        # the launching thread holds the GIL while it enqueues the steps: switch
        # threads often, or a short timed region gets a single sample
        self.switch = sys.getswitchinterval()
        sys.setswitchinterval(0.0001)
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        if self.nv is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            sys.setswitchinterval(self.switch)

    def _stats(self, rows):
        reasons = sorted({n for _, _, bits in rows for n, bit in self.REASONS.items() if bits & bit})
        return (statistics.median([m for _, m, _ in rows]) if rows else None), reasons, len(rows)

    def summary(self):
        t0, t1 = self.marks.get("start", float("-inf")), self.marks.get("end", float("inf"))
        timed = [r for r in self.samples if t0 <= r[0] <= t1]
        mhz, reasons, n = self._stats(timed)
        out = {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": n}
        if len(self.samples) > len(timed):
            mhz_all, reasons_all, n_all = self._stats(self.samples)
            out["with_following_steps"] = {"sm_mhz": mhz_all, "reasons": reasons_all,
                                           "samples": n_all}
        if self.err:
            out["note"] = self.err
        return out


def _dist(backend="nccl"):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws == 1:
        return None, 0, 1, 0
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return dist, dist.get_rank(), ws, int(os.environ.get("LOCAL_RANK", "0"))


def replica_inputs(wl, rank):
    """Inputs of one replica: the weights are the workload's (shared by every
    rank), the activations and routing are seeded by seed + rank."""
    import synth
    wl_r = wl if rank == 0 else synth.Workload(**{**wl.__dict__, "seed": wl.seed + rank})
    x, x_sf, idx, tw = synth.make_activations(wl_r)
    w1, w1_sf, w2, w2_sf = synth.make_weights(wl)
    return dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)


def max_over_ranks(v, dist, device):
    """The largest of every rank's v (one all-reduce; the value itself at N = 1)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _workload_desc(wl):
    return (f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} top{wl.k} "
            f"(W1 [{wl.E},{2 * wl.I},{wl.H}], W2 [{wl.E},{wl.H},{wl.I}] FP4 E2M1 + UE8M0/1x32; "
            f"x FP8 E4M3 + UE8M0/1x32)")


# ------------------------------------------------------------- CPU oracle
def _oracle_sample(wl, inputs, seconds: float, rng_seed=0):
    """Time the oracle on a bounded token sample; returns (TFLOPS, tokens, s, cores)."""
    import numpy as np

    import oracle
    cores = oracle.max_threads()
    rng = np.random.default_rng(rng_seed)
    n = max(2, min(wl.T, cores))
    toks = rng.choice(wl.T, n, replace=False).astype(np.int32)
    t0 = time.perf_counter()
    oracle.moe_forward(**inputs, tokens=toks)
    dt = time.perf_counter() - t0
    n2 = int(min(wl.T, max(n, n * seconds / max(dt, 1e-6))))
    if n2 > n:
        toks = rng.choice(wl.T, n2, replace=False).astype(np.int32)
        t0 = time.perf_counter()
        oracle.moe_forward(**inputs, tokens=toks)
        dt = time.perf_counter() - t0
        n = n2
    flops = 6.0 * n * wl.k * wl.H * wl.I
    return flops / dt / 1e12, n, dt, cores


def run_reference(args, wl, rank):
    """The reference arm: the CPU oracle, as it stands, on a bounded sample."""
    if rank != 0:
        return
    import numpy as np

    import oracle
    import synth
    inputs = synth.make_inputs(wl)
    cores = oracle.max_threads()
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    # calibrate a per-step token sample
    rng = np.random.default_rng(0)
    n = max(2, min(wl.T, cores))
    t0 = time.perf_counter()
    oracle.moe_forward(**inputs, tokens=rng.choice(wl.T, n, replace=False).astype(np.int32))
    dt = time.perf_counter() - t0
    n = int(min(wl.T, max(2, n * per_step / max(dt, 1e-6))))
    times = []
    for i in range(args.warmup + args.steps):
        toks = rng.choice(wl.T, n, replace=False).astype(np.int32)
        t0 = time.perf_counter()
        oracle.moe_forward(**inputs, tokens=toks)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = statistics.mean(times)
    flops = 6.0 * n * wl.k * wl.H * wl.I
    value = flops / sec / 1e12
    sample = f"{n} random tokens of {wl.T} per step (all their top-{wl.k} slots)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "tokens_per_s": n / sec, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": _workload_desc(wl)},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ ours
# The headline workload (the largest config: the Mega MoE usage-example shape) and
# the other configs, each measured the same way and reported as a sub-record of the
# same JSON line.
HEADLINE = "usage"
SUB_WORKLOADS = ["mid", "skewed", "decode", "decode@T64", "decode@T32", "decode@T16"]
GEN_WEIGHTS = {}   # (E, H, I, seed) -> host weights (skewed and decode share one layer)


def _weights(wl):
    key = (wl.E, wl.H, wl.I, wl.seed)
    if key not in GEN_WEIGHTS:
        import synth
        GEN_WEIGHTS.clear()
        GEN_WEIGHTS[key] = synth.make_weights(wl)
    return GEN_WEIGHTS[key]


def _roofline(wl, inputs, g1_ms, step_ms, pk, traffic):
    """linear1's roofline (the slower of its FLOPs at the tensor peak and its
    algorithmic bytes at the HBM peak) and the whole step's."""
    import numpy as np
    tensor_peak = 2.0 * pk["bf16"]  # FP8-rate MMA = 2 x the measured bf16 rate
    hbm_peak = pk["hbm"]
    # Algorithmic bytes: the weights of the experts that receive rows (FP4 codes +
    # one UE8M0 byte per 32) are read once; activations, intermediate and output once.
    idx = inputs["topk_idx"]
    R_valid = int((idx >= 0).sum())
    touched = len(np.unique(idx[idx >= 0]))
    H, I = wl.H, wl.I
    w1_bytes = touched * (2 * I * H // 2 + 2 * I * H // 32)
    w2_bytes = touched * (H * I // 2 + H * I // 32)
    g1_flops = 4.0 * R_valid * H * I
    g1_bytes = w1_bytes + R_valid * (H + H // 32) + R_valid * (I + I // 32)
    step_bytes = (w1_bytes + w2_bytes + wl.T * (H + H // 32) + wl.T * wl.k * 8 + wl.T * H * 2)
    if g1_flops / (tensor_peak * 1e12) >= g1_bytes / (hbm_peak * 1e9):
        roof = {"bound": "tensor", "achieved": g1_flops / (g1_ms * 1e-3) / 1e12,
                "peak": tensor_peak, "unit": "TFLOP/s",
                "peak_note": f"2 x bf16 burst {pk['bf16']} TFLOP/s ({pk['src']})"}
    else:
        roof = {"bound": "hbm", "achieved": g1_bytes / (g1_ms * 1e-3) / 1e9, "peak": hbm_peak,
                "unit": "GB/s", "peak_note": f"copy bandwidth {hbm_peak} GB/s ({pk['src']})"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof.update(kernel="linear1 (moe_gemm_kernel<1>, normal and narrow tiles)",
                flops_per_launch=g1_flops, algorithmic_bytes_per_launch=g1_bytes,
                traffic=traffic, traffic_unit="bytes per launch (ncu dram read+write)")
    t_tensor = wl.flops / (tensor_peak * 1e12)
    t_hbm = step_bytes / (hbm_peak * 1e9)
    step = {"bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "roofline_ms": max(t_tensor, t_hbm) * 1e3, "frac": max(t_tensor, t_hbm) * 1e3 / step_ms,
            "tflops": wl.flops / (step_ms * 1e-3) / 1e12,
            "hbm_gbs": step_bytes / (step_ms * 1e-3) / 1e9,
            "algorithmic_bytes": step_bytes, "experts_touched": touched}
    return roof, step


def measure(args, wl, inputs, dev, dist, weights=None, e2e=True):
    """Time one workload: K replays of one captured plan + forward (L2 flushed
    before each), then K eager steps with events at the kernel boundaries,
    then (e2e) the host-buffer entry point.  Returns (record, layer)."""
    import numpy as np
    import torch

    import block_scaled_fp8_permute_b200 as moe
    from block_scaled_fp8_permute_b200.layer import MoELayer

    lay = MoELayer(inputs, device=dev, weights=weights)
    shp, d = lay.shape, lay.dev
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        moe.moe_plan(shp, d["topk_idx"], lay.ws)
        moe.moe_forward(shp, d["x"], d["x_sf"], d["topk_idx"], d["topk_w"], *lay.wt, lay.y,
                        lay.ws)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(lay.ws) == 0, "device status after warm-up"

    K = args.steps
    # One step (plan + forward) captured as a CUDA graph: the timed region replays it, so
    # the steps carry no host launch gaps and no events between kernels (which would
    # also break the programmatic-dependent-launch overlap of consecutive kernels).
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for row in kev:
        for e in row:
            e.record(stream)  # materialise the handles
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    # clocks: sampled over the timed region (marked) and, as more evidence for a short
    # region, over the eager kernel-timing steps that follow it
    clk = ClockSampler(torch.cuda.current_device())
    clk.__enter__()
    clk.wait_first()
    clk.mark("start")
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        graph.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clk.mark("end")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    del graph

    # Kernel durations: the same steps run eagerly with events at the kernel
    # boundaries (moe_set_timing_events), K more steps.
    for i in range(K):
        flush.zero_()
        kev[i][0].record(stream)
        moe.moe_set_timing_events(kev[i][1:6])
        step()
    moe.moe_set_timing_events(None)
    torch.cuda.synchronize()
    clk.__exit__(None, None, None)
    kern = {name: statistics.mean(kev[i][a].elapsed_time(kev[i][b]) for i in range(K))
            for name, a, b in (("plan", 0, 1), ("permute", 1, 2), ("linear1", 2, 3),
                               ("linear2", 3, 4), ("combine", 4, 5))}
    status = moe.moe_get_device_status(lay.ws)
    assert status == 0, f"device status {status}"
    rec = {"ms": statistics.mean(step_ms), "ms_p50": statistics.median(step_ms),
           "kernels_ms": kern, "clocks": clk.summary()}

    if e2e:
        # the host-buffer entry point, host<->device copies inside the timed region
        ws_h = moe.alloc_workspace(shp, dev, host_variant=True)
        pin = {k: torch.from_numpy(np.ascontiguousarray(inputs[k])).pin_memory()
               for k in ("x", "x_sf", "topk_idx", "topk_w")}
        y_host = torch.empty((wl.T, wl.H), dtype=torch.int16).pin_memory()
        e2e_ms = []
        for i in range(max(args.warmup, 3) + K):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            moe.moe_forward_host(shp, pin["x"], pin["x_sf"], pin["topk_idx"], pin["topk_w"],
                                 *lay.wt, y_host, ws_h)
            e1.record(stream)
            e1.synchronize()
            if i >= max(args.warmup, 3):
                e2e_ms.append(e0.elapsed_time(e1))
        rec["e2e_serial_ms"] = statistics.mean(e2e_ms)
        rec["h2d"] = sum(t.numel() * t.element_size() for t in pin.values())
        rec["d2h"] = y_host.numel() * y_host.element_size()
        del ws_h
        # the overlapped host-buffer call: K batches in one call, batch i + 1's
        # inputs going up and batch i - 1's y coming down while batch i computes
        ws_p = moe.alloc_workspace(shp, dev, host_variant="pipelined")
        y2 = [y_host, torch.empty_like(y_host).pin_memory()]

        def pipelined(n):
            moe.moe_forward_host_pipelined(shp, [pin["x"]] * n, [pin["x_sf"]] * n,
                                           [pin["topk_idx"]] * n, [pin["topk_w"]] * n, *lay.wt,
                                           [y2[i & 1] for i in range(n)], ws_p)
        flush.zero_()
        pipelined(max(args.warmup, 3))
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        pipelined(K)
        e1.record(stream)
        e1.synchronize()
        rec["e2e_ms"] = e0.elapsed_time(e1) / K
        del ws_p, y2
    del flush
    return rec, lay


def _launches_per_step(wl):
    # count+scan, scatter, permute, linear1, linear2, combine; with narrow tiles (the
    # library's default when the layer has <= 128 rows per expert) a second linear1
    # and linear2 launch run the narrow m-tiles
    return 6 + (2 if wl.R <= 128 * wl.E else 0)


def _cpu_baseline(wl, inputs, seconds):
    cv, n, sec, cores = _oracle_sample(wl, inputs, seconds)
    return {"value": cv, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
            "tokens_per_s": n / sec,
            "sample": f"{n} random tokens of {wl.T} (all top-{wl.k} slots), {sec:.1f} s"}


def sub_record(args, wl, pk):
    """One config measured at N = 1 as a sub-record of the headline line."""
    import gc

    import torch
    x, x_sf, idx, tw = __import__("synth").make_activations(wl)
    w1, w1_sf, w2, w2_sf = _weights(wl)
    inputs = dict(x=x, x_sf=x_sf, topk_idx=idx, topk_w=tw, w1=w1, w1_sf=w1_sf, w2=w2, w2_sf=w2_sf)
    key = (wl.E, wl.H, wl.I, wl.seed)
    wt = SUB_DEVICE_WEIGHTS.get(key)
    lay_inputs = dict(inputs, E=wl.E, I=wl.I) if wt is not None else inputs
    rec, lay = measure(args, wl, lay_inputs, "cuda:0", None, weights=wt, e2e=True)
    SUB_DEVICE_WEIGHTS.clear()
    SUB_DEVICE_WEIGHTS[key] = lay.wt
    roof, step = _roofline(wl, inputs, rec["kernels_ms"]["linear1"], rec["ms"], pk,
                           _linear1_traffic(wl.name))
    out = {"workload": _workload_desc(wl), "ms_per_step": rec["ms"], "ms_p50": rec["ms_p50"],
           "tflops": wl.flops / (rec["ms"] * 1e-3) / 1e12,
           "tokens_per_s": wl.T / (rec["ms"] * 1e-3), "roofline": roof, "step_roofline": step,
           "kernels_ms": rec["kernels_ms"], "clocks": rec["clocks"],
           "e2e": {"value": wl.flops / (rec["e2e_ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
                   "ms_per_step": rec["e2e_ms"], "h2d_bytes_per_step": rec["h2d"],
                   "d2h_bytes_per_step": rec["d2h"], "mode": "pipelined",
                   "serial_ms_per_step": rec["e2e_serial_ms"]},
           "gpu_launches_per_step": _launches_per_step(wl)}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = _cpu_baseline(wl, inputs, args.sub_cpu_seconds)
    del lay
    gc.collect()
    torch.cuda.empty_cache()
    return out


SUB_DEVICE_WEIGHTS = {}


def run_ours(args, wl, dist, rank, world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    inputs = replica_inputs(wl, rank)  # shared weights, this replica's activations / routing
    rec, lay = measure(args, wl, inputs, dev, dist)
    ms = max_over_ranks(rec["ms"], dist, dev)
    e2e = max_over_ranks(rec["e2e_ms"], dist, dev)
    e2e_serial = max_over_ranks(rec["e2e_serial_ms"], dist, dev)
    g1 = max_over_ranks(rec["kernels_ms"]["linear1"], dist, dev)
    del lay
    subs = {}
    if world == 1 and args.workload is None and not args.no_sub:
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        pk = _peaks()
        for name in SUB_WORKLOADS:
            subs[name] = sub_record(args, __import__("synth").workload(name), pk)
    if rank != 0:
        return
    flops = wl.flops * world
    value = flops / (ms * 1e-3) / 1e12
    pk = _peaks()
    roof, step = _roofline(wl, inputs, g1, ms / 1.0, pk, _linear1_traffic(wl.name))
    if world > 1:  # the step roofline of one replica (every rank runs the same shape)
        step["note"] = "per replica"
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = _cpu_baseline(wl, inputs, args.cpu_seconds)
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOPS",
        "tokens_per_s": wl.T * world / (ms * 1e-3),
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3 x fp4_e2m1, fp32 accumulate, bf16 out", "data": "synthetic",
        "config": {"workload": _workload_desc(wl), "tokens_per_gpu": wl.T,
                   "l2": "flushed (256 MB write) before every timed step",
                   "step": "moe_plan + moe_forward replayed as one CUDA graph",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "kernels_ms": rec["kernels_ms"],
        "kernels_ms_note": "eager steps with events at kernel boundaries (K extra steps)",
        "step_roofline": step,
        "e2e": {"value": flops / (e2e * 1e-3) / 1e12, "unit": "TFLOPS",
                "h2d_bytes_per_step": rec["h2d"], "d2h_bytes_per_step": rec["d2h"],
                "ms_per_step": e2e,
                "mode": ("moe_forward_host_pipelined over the K steps (pinned host buffers; "
                         "step i+1's inputs up and step i-1's y down while step i computes)"),
                "serial_ms_per_step": e2e_serial,
                "serial_note": "moe_forward_host, one synchronous call per step"},
        "gpu_launches": _launches_per_step(wl) * args.steps,
        "clocks": rec["clocks"],
        "cpu_baseline": cpu,
    }
    if subs:
        out["configs"] = subs
        out["configs_note"] = ("the other configs, each measured at N = 1 like the headline "
                               "(graph-replayed step, L2 flushed, CUDA events)")
    print(json.dumps(out), flush=True)


# ------------------------------------------------- standalone FP8 x FP4 GEMM
# name -> (G, M or M_max, N, K, masked): a prefill-sized dense projection, a small one,
# and a decode-style masked grouped GEMM (16 groups, 1..64 rows each, weights read once)
GEMM_SHAPES = {"gemm": (1, 4096, 7168, 7168, False), "gemm-small": (1, 512, 2048, 1024, False),
               "gemm-masked": (16, 128, 4096, 7168, True)}


def run_gemm(args, name):
    """The standalone GEMM: K timed replays of one captured call, L2 flushed
    before each, one JSON line."""
    import numpy as np
    import torch

    import block_scaled_fp8_permute_b200 as moe
    import synth

    G, M, N, K, masked = GEMM_SHAPES[name]
    a, a_sf = synth.make_x(G * M, K, 0)
    b, b_sf = synth.make_w(G, N, K, 2, 0)
    counts = (np.random.default_rng(0).integers(1, 65, G).astype(np.int32) if masked
              else np.full(G, M, np.int32))
    dev = "cuda:0"
    da = torch.from_numpy(a).to(dev)
    das = torch.from_numpy(a_sf).to(dev)
    b_t, b_sf_t = moe.gemm_transform_b(G, N, K, torch.from_numpy(b).to(dev),
                                       torch.from_numpy(b_sf).to(dev))
    d = torch.empty((G * M, N), dtype=torch.int16, device=dev)
    mm = torch.from_numpy(counts).to(dev)
    ws = moe.alloc_gemm_workspace(G, M, N, K, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        if masked:
            moe.moe_gemm_fp8_fp4_masked(G, M, N, K, da, das, mm, b_t, b_sf_t, d, ws)
        else:
            moe.moe_gemm_fp8_fp4(M, N, K, da, das, b_t, b_sf_t, d, ws)

    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call()
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    K_ = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_)]
    with ClockSampler(0) as clk:
        clk.wait_first()
        clk.mark("start")
        for i in range(K_):
            flush.zero_()
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        clk.mark("end")
    ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K_))
    rows = int(counts.sum())
    flops = 2.0 * rows * N * K
    algo_bytes = (rows * (K + K // 32) + G * (N * K // 2 + N * (K // 32)) + rows * N * 2)
    pk = _peaks()
    tpeak, hpeak = 2.0 * pk["bf16"], pk["hbm"]
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    if flops / (tpeak * 1e12) >= algo_bytes / (hpeak * 1e9):
        roof = {"bound": "tensor", "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s",
                "peak_note": f"2 x bf16 burst {pk['bf16']} TFLOP/s ({pk['src']})"}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": hpeak, "unit": "GB/s",
                "peak_note": f"copy bandwidth {hpeak} GB/s ({pk['src']})"}
    roof.update(frac=roof["achieved"] / roof["peak"], kernel="moe_gemm_kernel<3>",
                flops_per_launch=flops, algorithmic_bytes_per_launch=algo_bytes, traffic=None)
    del graph
    shape = (f"G={G} M_max={M} (rows {rows}) N={N} K={K}" if masked else f"M={M} N={N} K={K}")
    print(json.dumps({
        "metric": "FP8xFP4 GEMM TFLOPS on 1 B200 (standalone, BF16 out)", "value": tflops,
        "unit": "TFLOPS", "gbs": gbs, "n_gpus": 1, "steps": K_, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3 x fp4_e2m1, fp32 accumulate, bf16 out", "data": "synthetic",
        "config": {"workload": f"{name}: {shape}", "l2": "flushed before every step",
                   "step": "one GEMM call replayed as a CUDA graph"},
        "roofline": roof,
        "gpu_launches": 3 * K_,  # tile list, scale chunks, GEMM
        "clocks": clk.summary(), "cpu_baseline": None}), flush=True)


# ------------------------------------------------------- FP4 indexer (MQA logits)
def run_indexer(args, name):
    """The FP4 indexer: K timed replays of one captured call (key layout and
    scale chunks rebuilt inside the call), L2 flushed before each, one JSON line."""
    import numpy as np
    import torch

    import block_scaled_fp8_permute_b200 as moe
    import oracle
    import synth

    wl = synth.INDEXER_WORKLOADS[name]
    d = synth.make_indexer(wl.S, wl.Hh, wl.D, wl.N, wl.seed)
    dev = "cuda:0"
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for k, v in d.items()}
    out = torch.empty((wl.S, wl.N), dtype=torch.float32, device=dev)
    ws = moe.alloc_mqa_workspace(wl.S, wl.Hh, wl.D, wl.N, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        moe.moe_fp8_fp4_mqa_logits(t["q"], t["q_sf"], t["kv"], t["kv_sf"], t["weights"], t["ks"],
                                   t["ke"], out, ws)

    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        call()
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(0) as clk:
        clk.wait_first()
        clk.mark("start")
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        clk.mark("end")
    ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))
    del graph
    S, Hh, D, N = wl.S, wl.Hh, wl.D, wl.N
    algo_bytes = (S * Hh * (D + D // 32) + N * (D // 2 + D // 32) + S * Hh * 4 + S * 8
                  + S * N * 4)
    pk = _peaks()
    tpeak, hpeak = 2.0 * pk["bf16"], pk["hbm"]
    tflops = wl.flops / (ms * 1e-3) / 1e12
    gbs = algo_bytes / (ms * 1e-3) / 1e9
    if wl.flops / (tpeak * 1e12) >= algo_bytes / (hpeak * 1e9):
        roof = {"bound": "tensor", "achieved": tflops, "peak": tpeak, "unit": "TFLOP/s",
                "peak_note": f"2 x bf16 burst {pk['bf16']} TFLOP/s ({pk['src']})"}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": hpeak, "unit": "GB/s",
                "peak_note": f"copy bandwidth {hpeak} GB/s ({pk['src']})"}
    roof.update(frac=roof["achieved"] / roof["peak"], kernel="mqa_logits_kernel",
                flops_per_launch=wl.flops, algorithmic_bytes_per_launch=algo_bytes, traffic=None)
    cpu = None
    if not args.no_cpu_baseline:
        rows = np.arange(min(S, 8), dtype=np.int64)
        sub = dict(d)
        for k in ("q", "q_sf", "weights", "ks", "ke"):
            sub[k] = np.ascontiguousarray(d[k][rows])
        t0 = time.perf_counter()
        oracle.mqa_logits(**sub)
        sec = time.perf_counter() - t0
        pairs = int(sum(max(0, min(int(sub["ke"][r]), N) - max(int(sub["ks"][r]), 0))
                        for r in range(len(rows))))
        cpu = {"value": 2.0 * Hh * D * pairs / sec / 1e12, "unit": "TFLOPS",
               "cores": oracle.max_threads(), "kind": "oracle",
               "sample": f"{len(rows)} query rows of {S} (all their keys), {sec:.1f} s"}
    print(json.dumps({
        "metric": "FP4-indexer MQA logits TFLOPS on 1 B200 (FP8 q x FP4 k, FP32 logits)",
        "value": tflops, "unit": "TFLOPS", "gbs": gbs, "n_gpus": 1, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8_e4m3 x fp4_e2m1, fp32 accumulate, fp32 out",
        "data": "synthetic",
        "config": {"workload": f"{name}: S={S} Hh={Hh} D={D} N={N}, query i sees keys "
                               f"[0, N - S + i + 1)", "l2": "flushed before every step",
                   "step": "one call replayed as a CUDA graph (key layout rebuilt inside)"},
        "roofline": roof,
        "gpu_launches": 3 * K,  # key layout, query scale chunks, logits
        "clocks": clk.summary(), "cpu_baseline": cpu}), flush=True)


def main():
    args = _args()
    import synth
    if args.workload in synth.INDEXER_WORKLOADS:
        if int(os.environ.get("RANK", "0")) == 0 and args.impl == "ours":
            run_indexer(args, args.workload)
        return
    if args.workload in GEMM_SHAPES:
        if int(os.environ.get("RANK", "0")) == 0 and args.impl == "ours":
            run_gemm(args, args.workload)
        return
    wl = synth.workload(args.workload or HEADLINE)
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; other ranks leave at once
        run_reference(args, wl, int(os.environ.get("RANK", "0")))
        return
    dist, rank, world, local_rank = _dist()
    if args.gemm_variant is not None or args.swap_max is not None or args.narrow is not None:
        import block_scaled_fp8_permute_b200 as moe
        if args.gemm_variant is not None:
            moe.moe_set_gemm_variant(args.gemm_variant)
        if args.swap_max is not None:
            moe.moe_set_swap_max(args.swap_max)
        if args.narrow is not None:
            moe.moe_set_narrow_tiles(args.narrow)
    try:
        run_ours(args, wl, dist, rank, world, local_rank)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
