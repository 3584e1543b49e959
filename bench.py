#!/usr/bin/env python
"""Benchmark of the fused NA2D forward (queries*heads per second).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one ``na2d_forward`` call per shape of the workload over one batch
of synthetic input (default: the NAT-Tiny stage-1 shape, B=32 heads=2 56x56
D=32 k=7 d=1, fp16).  Inputs are resident in HBM before timing; between steps
the benchmark rotates through enough distinct input/output sets that their
total exceeds 3x the L2 cache, so every step reads from HBM.  Steps are
replayed from CUDA graphs and timed with CUDA events on the launching stream.

For N > 1 (launched by torch.distributed.run) every rank processes its own
batch (weak scaling, no collective on the data path); the time is the maximum
over ranks.

``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload.
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
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from dataclasses import replace  # noqa: E402

from neighborhood_attention_na2d_b200.inputs import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "NA2D forward queries·heads/sec (GB/s, % HBM roofline) at NAT/DiNAT shapes"
UNIT = "queries*heads/s"
FALLBACK_HBM_GBS = 6650.0
PEAKS_FILE = ROOT / "MEASURED_PEAKS.json"
PROFILES = ROOT / "profiles"
CSRC = "neighborhood_attention_na2d_b200/csrc/"
# The sources each profiled kernel is built from (device code and the host
# code that plans and launches it).
KERNEL_SOURCES = {
    "fwd_stream_kernel": [CSRC + "na2d_stream.cu", CSRC + "na2d_device.cuh", CSRC + "na2d_launch.h"],
    "fwd_umma_kernel": [CSRC + "na2d_umma.cu", CSRC + "na2d_tc.cu", CSRC + "na2d_tcgen05.cuh", CSRC + "na2d_device.cuh",
                        CSRC + "na2d_launch.h"],
    "fwd_ugrp_kernel": [CSRC + "na2d_ugrp.cu", CSRC + "na2d_tc.cu", CSRC + "na2d_tcgen05.cuh", CSRC + "na2d_device.cuh",
                        CSRC + "na2d_launch.h"],
    "fwd_tc_kernel": [CSRC + "na2d_tc.cu", CSRC + "na2d_device.cuh", CSRC + "na2d_launch.h"],
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def code_only(text: str) -> str:
    """C++ source without comments and blank lines, so that an edit of the
    comments alone does not count as a kernel change."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_sha(kernel: str) -> str:
    """Hash of a kernel's sources without their comments."""
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        h.update(code_only((ROOT / p).read_text()).encode())
    return h.hexdigest()[:16]


def hbm_peak() -> tuple[float, str]:
    try:
        d = json.loads(PEAKS_FILE.read_text())
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel: str, workload: str) -> int | None:
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, only if it was taken on the current kernel source.  A
    kernel name with a mode suffix ("fwd_tc_kernel/full") is looked up by the
    kernel's name."""
    kernel = kernel.split("/")[0]
    f = PROFILES / f"{kernel}_{workload}.md"
    if not f.exists() or kernel not in KERNEL_SOURCES:
        return None
    text = f.read_text()
    m = re.search(r"traffic_per_launch_bytes\s*=\s*(\d+)\s*;\s*kernel_sha\s*=\s*([0-9a-f]+)", text)
    if not m or m.group(2) != kernel_sha(kernel):
        return None
    return int(m.group(1))


# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            log(f"clock sampling unavailable: {e}")
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_reasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            self._stop.wait(0.01)

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
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def workload(args):
    """The selected workload, with B overridden by --batch if given."""
    wl = WORKLOADS[args.workload]
    if args.batch:
        wl = replace(wl, name=f"{wl.name}_B{args.batch}",
                     shapes=tuple(replace(s, B=args.batch) for s in wl.shapes))
    return wl


# ---------------------------------------------------------------------------
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        log(f"--gpus {args.gpus} but WORLD_SIZE {world}: using WORLD_SIZE")
    return world, rank, local


def max_over_ranks(x: float, pg, dev) -> float:
    """The largest of every rank's x (every rank calls this at the same point,
    so all of them take the same collective steps); x itself on one rank."""
    if not pg:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, world, rank):
    """The oracle on host cores, per step a bounded sample of the workload."""
    if rank != 0:
        return
    import oracle

    wl = workload(args)
    threads = oracle.default_threads()
    # sample: the first nb batch elements of every shape -- enough (batch, head)
    # slices to occupy every host core; the step count is cut below if needed
    # so the run stays within minutes
    nb = max(1, min(min(s.B for s in wl.shapes), math.ceil(threads / min(s.heads for s in wl.shapes))))
    threads = min(threads, nb * min(s.heads for s in wl.shapes))
    arrays = [[t[:nb].double().numpy() if t.dim() == 5 else t.double().numpy() for t in make_inputs(s)]
              for s in wl.shapes]
    def step():
        for s, (qq, kk, vv, rr) in zip(wl.shapes, arrays):
            oracle.forward(qq, kk, vv, rr, s.k, s.d, nthreads=threads)
    t0 = time.perf_counter()
    step()
    one = time.perf_counter() - t0
    budget = 150.0
    steps, warmup = args.steps, args.warmup
    if (steps + warmup) * one > budget:
        steps = max(1, int(budget / one) - warmup)
        warmup = min(warmup, 3)
    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / steps
    units = sum(nb * s.heads * s.H * s.W for s in wl.shapes)
    value = units / dt
    sample = f"first {nb} batch element(s) of each shape ({units} query*heads per step), fp64, all-host-core oracle"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    if steps != args.steps:
        line["note"] = f"steps reduced from {args.steps} to fit the CPU time budget"
    print(json.dumps(line), flush=True)


def config_dict(wl, world):
    s0 = wl.shapes[0]
    cfg = {"workload": wl.name, "shapes": [s.describe() for s in wl.shapes],
           "B": s0.B, "heads": s0.heads, "H": s0.H, "W": s0.W, "D": s0.D, "k": s0.k, "d": s0.d,
           "global_batch": s0.B * world, "parallelism": f"replicas{world}" if world > 1 else "single"}
    return cfg


def cpu_baseline(wl):
    """The oracle as it stands on all host cores, one pass over a bounded sample."""
    import oracle
    threads = oracle.default_threads()
    total_units, total_t = 0, 0.0
    parts = []
    for s in wl.shapes:
        q, k, v, rpb = make_inputs(s)
        nb = s.B
        # bound the sample to about 10 s of CPU work: ~5 us of fp64 work per key*query on one core
        est = s.B * s.heads * s.H * s.W * s.k * s.k * 5e-8
        if est > 10.0:
            nb = max(1, int(s.B * 10.0 / est))
        arr = [t[:nb].double().numpy() for t in (q, k, v)] + [rpb.double().numpy()]
        t0 = time.perf_counter()
        oracle.forward(*arr, s.k, s.d, nthreads=threads)
        total_t += time.perf_counter() - t0
        total_units += nb * s.heads * s.H * s.W
        parts.append(f"{nb}/{s.B} batch of {s.describe()}")
    used = min(threads, min(s.B * s.heads for s in wl.shapes))
    return {"value": total_units / total_t, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": "; ".join(parts) + "; one pass, fp64"}


def graph_plan(K: int, G_max: int = 200) -> tuple[int, int, int]:
    """How K timed steps are split into CUDA-graph replays: a graph of G steps
    replayed `full` times, then a graph of `rest` steps (rest < G), so that one
    timed run is exactly K steps."""
    if K < 1:
        raise ValueError("--steps must be at least 1")
    G = min(K, G_max)
    full, rest = divmod(K, G)
    return G, full, rest


def make_sets(wl, dev, rank, l2):
    """Resident input/output sets, rotated so that every step misses L2."""
    import torch
    elem = {"f32": 4, "f16": 2, "bf16": 2}
    set_bytes = sum(4 * s.B * s.heads * s.H * s.W * s.D * elem[s.dtype] for s in wl.shapes)
    R = max(2, math.ceil(3 * l2 / set_bytes))
    sets = []
    for r in range(R):
        one = []
        for s in wl.shapes:
            q, k, v, rpb = make_inputs(s, s.seed + 1000 * r + 100000 * rank)
            q, k, v, rpb = (t.to(dev) for t in (q, k, v, rpb))
            one.append((s, q, k, v, rpb, torch.empty_like(q)))
        sets.append(one)
    torch.cuda.synchronize()
    return sets, set_bytes


def time_steps(wl, sets, K, warmup, dev, pg=None, min_seconds=0.25, min_runs=5, clocks=None):
    """Times K steps of the workload (one na2d_forward per shape per step,
    rotating the input sets).  The K steps are replayed from CUDA graphs (see
    graph_plan) between CUDA events on the launching stream, bracketed by a
    barrier and device synchronisation; the run is repeated until about
    min_seconds have been timed and the median run is returned, as ms per step,
    with the run count and the spread."""
    import torch
    import neighborhood_attention_na2d_b200 as na

    R = len(sets)

    def step(i):
        for (s, q, k, v, rpb, out) in sets[i % R]:
            na.na2d_forward(q, k, v, rpb, s.k, s.d, out=out)

    for i in range(max(warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    G, full, rest = graph_plan(K)
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    graphs = []
    with torch.cuda.stream(stream):
        for n in ([G] + ([rest] if rest else [])):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(i)
            graphs.append(g)
        torch.cuda.synchronize()
        for g in graphs:      # one untimed replay of each graph
            g.replay()
        torch.cuda.synchronize()
        runs = []
        t_total = 0.0
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx = clocks if clocks is not None else _Null()
        with ctx:
            while len(runs) < min_runs or t_total < min_seconds * 1e3:
                if pg:
                    pg.barrier()
                torch.cuda.synchronize()
                start.record(stream)
                for _ in range(full):
                    graphs[0].replay()
                if rest:
                    graphs[1].replay()
                end.record(stream)
                end.synchronize()
                ms = max_over_ranks(start.elapsed_time(end), pg, dev)
                runs.append(ms)
                t_total += ms
                if len(runs) >= 10000:
                    break
    torch.cuda.synchronize()
    del graphs
    med = statistics.median(runs)
    return {"ms_per_step": med / K, "runs": len(runs), "graph_steps": G, "replays_per_run": full + (1 if rest else 0),
            "min_ms_per_step": min(runs) / K, "max_ms_per_step": max(runs) / K}


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


def tensor_peak() -> tuple[float, str]:
    """Dense bf16 tensor peak (TFLOP/s) from MEASURED_PEAKS.json (burst figure;
    fp16 runs at the same rate)."""
    try:
        d = json.loads(PEAKS_FILE.read_text())
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def step_traffic(kerns, workload: str) -> int | None:
    """Recorded DRAM bytes of one step: the one kernel's per-launch figure, or
    the sum over the shapes' kernels when each shape runs a different kernel
    (each has its own summary for this workload); None if any is missing."""
    if not kerns:
        return None
    if isinstance(kerns, str):
        kerns = [kerns]
    if len(set(kerns)) != len(kerns):
        return None
    got = [recorded_traffic(k, workload) for k in kerns]
    return None if any(g is None for g in got) else sum(got)


def roofline(wl, ms_per_step, kern):
    """Roofline of one step: the slower of the algorithmic bytes at the HBM
    peak and the useful FLOPs at the tensor peak; achieved is measured against
    that bound."""
    alg_bytes = sum(s.algorithmic_bytes() for s in wl.shapes)
    flops = sum(s.useful_flops() for s in wl.shapes)
    hbm, hbm_kind = hbm_peak()
    tc, tc_kind = tensor_peak()
    t_hbm = alg_bytes / (hbm * 1e9)
    t_tc = flops / (tc * 1e12)
    sec = ms_per_step / 1e3
    if t_hbm >= t_tc:
        achieved = alg_bytes / sec / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_source": f"{hbm_kind} hbm_gbs (copy)"}
    else:
        achieved = flops / sec / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc, "unit": "TFLOP/s", "frac": achieved / tc,
                "peak_source": f"{tc_kind} bf16_tflops (burst)"}
    roof.update({"traffic": step_traffic(kern, wl.name),
                 "algorithmic_bytes_per_step": alg_bytes, "useful_flops_per_step": flops,
                 "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6, "kernel": kern})
    return roof


def run_ours(args, world, rank, local):
    import torch
    import neighborhood_attention_na2d_b200 as na

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    na.lib()
    wl = workload(args)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    sets, set_bytes = make_sets(wl, dev, rank, l2)
    R = len(sets)
    log(f"rank {rank}: {R} input sets x {set_bytes / 1e6:.1f} MB (L2 {l2 / 1e6:.0f} MB)")
    K = args.steps
    clocks = ClockSampler(local)
    t = time_steps(wl, sets, K, args.warmup, dev, pg, clocks=clocks)
    ms_per_step = t["ms_per_step"]
    units_rank = sum(s.B * s.heads * s.H * s.W for s in wl.shapes)
    value = world * units_rank / (ms_per_step / 1e3)
    kern = kernels_of(wl)
    roof = roofline(wl, ms_per_step, kern[0] if len(set(kern)) == 1 else kern)
    del sets

    # ---- the other workloads of the same problem, each timed the same way (1 GPU)
    per_wl = {}
    if world == 1 and not args.no_per_workload:
        for name in PER_WORKLOAD:
            if name == wl.name:
                continue
            w2 = WORKLOADS[name]
            s2, _ = make_sets(w2, dev, rank, l2)
            t2 = time_steps(w2, s2, K, args.warmup, dev, None)
            k2 = kernels_of(w2)
            r2 = roofline(w2, t2["ms_per_step"], k2[0] if len(set(k2)) == 1 else k2)
            per_wl[name] = {"ms_per_step": t2["ms_per_step"],
                            "value": sum(s.B * s.heads * s.H * s.W for s in w2.shapes) / (t2["ms_per_step"] / 1e3),
                            "frac": r2["frac"], "bound": r2["bound"], "achieved": r2["achieved"],
                            "traffic": r2["traffic"], "kernels": k2, "shapes": [s.describe() for s in w2.shapes],
                            "runs": t2["runs"]}
            del s2
        torch.cuda.empty_cache()

    # ---- the other calls of the library on NAT-Tiny stage-1-sized inputs (1 GPU)
    ext = {}
    if world == 1 and not args.no_per_workload:
        ext = time_extensions(dev, l2, args.warmup)
        torch.cuda.empty_cache()

    # ---- end to end through the public API: pinned host -> device, forward, device -> host
    e2e = run_e2e(args, wl, dev, rank, world, pg)

    cfg = config_dict(wl, world)
    cfg.update({"l2": f"rotating {R} input sets ({R * set_bytes / 1e6:.0f} MB) > 3x L2 ({l2 / 1e6:.0f} MB)",
                "timing": (f"each timed run is exactly {K} steps: a CUDA graph of {t['graph_steps']} steps "
                           f"replayed {t['replays_per_run']} time(s) (a second graph holds the remainder); "
                           f"CUDA events on the launching stream; median of {t['runs']} runs"),
                "ms_per_step_min_max": [t["min_ms_per_step"], t["max_ms_per_step"]]})
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.shapes[0].dtype, "data": "synthetic (seeded N(0,1) q/k/v, N(0,0.02) rpb)", "config": cfg,
        "roofline": roof, "e2e": e2e, "gpu_launches": K * len(wl.shapes), "clocks": clocks.summary(),
    }
    if per_wl:
        line["per_workload"] = per_wl
    if ext:
        line["extensions"] = ext
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_calls(fn, n_sets, warmup, dev, min_seconds=0.2):
    """Median time of one call of fn(i) (i rotates over n_sets input sets),
    replayed from a CUDA graph of 20 calls, CUDA events on the stream."""
    import torch
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(20):
                fn(i)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        runs, total = [], 0.0
        while len(runs) < 5 or total < min_seconds * 1e3:
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            ms = a.elapsed_time(b)
            runs.append(ms / 20)
            total += ms
    torch.cuda.synchronize()
    del g
    return statistics.median(runs)


def time_extensions(dev, l2, warmup):
    """Times the library's other calls at the NAT-Tiny stage-1 size (B=32,
    heads=2, 56x56, D=32, k=7, d=1; fp16 unless noted), rotating input sets
    beyond 3x L2: the backward; the forward read in place from a channels-last
    fused q/k/v buffer; the forward returning the attention weights with
    dropout p=0.1; a D=64 forward (heads=1 so the bytes match); a map
    shorter than k*d (DiNAT stage-4-sized 7x7 with dilation 2, padded to
    14x14, B=128 heads=16 bf16).  HBM fraction against the measured copy
    bandwidth, on the bytes each call must move."""
    import torch
    import neighborhood_attention_na2d_b200 as na
    from neighborhood_attention_na2d_b200.inputs import Shape

    peak, _ = hbm_peak()
    out = {}
    nat = Shape(32, 2, 56, 56, 32, 7, 1, "f16", 1)
    qh = nat.queries_heads
    tensor = qh * 64                                          # one [B,heads,H,W,32] fp16 tensor

    def sets(shape, n_extra=0):
        R = max(2, math.ceil(3 * l2 / (4 * shape.queries_heads * shape.D * 2)))
        res = []
        for r in range(R):
            q, k, v, rpb = (t.to(dev) for t in make_inputs(shape, shape.seed + 1000 * r))
            res.append([q, k, v, rpb] + [torch.randn_like(q) for _ in range(n_extra)])
        return res

    def record(name, shape, ms, moved, kernel, note):
        out[name] = {"ms_per_call": ms, "value": shape.queries_heads / (ms / 1e3), "unit": UNIT,
                     "achieved_gbs": moved / (ms / 1e3) / 1e9, "frac": moved / (ms / 1e3) / 1e9 / peak,
                     "bytes_per_call": moved, "kernel": kernel, "shape": shape.describe(), "note": note}

    # backward
    S = sets(nat, 1)
    ws = torch.empty(na.backward_workspace_size(na.make_problem(S[0][0].shape, 7, 1, S[0][0].dtype)),
                     dtype=torch.uint8, device=dev)
    grads = [torch.empty_like(S[0][0]) for _ in range(3)] + [torch.empty_like(S[0][3])]

    def bwd(i):
        q, k, v, rpb, g = S[i % len(S)]
        na.na2d_backward(q, k, v, rpb, g, 7, 1, *grads, workspace=ws)
    ms = time_calls(bwd, len(S), warmup, dev)
    record("backward", nat, ms, 7 * tensor + 2 * 8 * qh, na.na2d_last_kernel(),
           "reads q, k, v, dout; writes dq, dk, dv; 8 bytes per query of statistics written and read")
    del S, ws, grads

    # channels-last fused q/k/v, read in place
    R = max(2, math.ceil(3 * l2 / (4 * tensor)))
    bufs = [(torch.randn(32, 56, 56, 3 * 2 * 32, device=dev).half(), torch.empty(32, 56, 56, 64, device=dev).half())
            for _ in range(R)]
    rpb = (torch.randn(2, 13, 13, device=dev) * 0.02).half()

    def qkv(i):
        x, o = bufs[i % R]
        na.na2d_qkv_packed(x, rpb, 7, 1, 2, out=o)
    ms = time_calls(qkv, R, warmup, dev)
    record("fused_qkv_channels_last", nat, ms, 4 * tensor, na.na2d_last_kernel(),
           "q, k, v strided views of one (B, H, W, 3*heads*D) buffer, output (B, H, W, heads*D)")
    del bufs

    # weights out + dropout
    S = sets(nat)
    outs = torch.empty_like(S[0][0])

    def wdrop(i):
        q, k, v, rpb = S[i % len(S)]
        na.na2d_forward_ex(q, k, v, rpb, 7, 1, out=outs, return_attn=True, dropout_p=0.1, seed=i)
    ms = time_calls(wdrop, len(S), warmup, dev)
    record("weights_and_dropout", nat, ms, 4 * tensor + qh * 49 * 4, na.na2d_last_kernel(),
           "attention dropout p=0.1 (Philox mask) and the fp32 weights [B, heads, H, W, 49] written")
    del S, outs

    # D = 64
    d64 = Shape(32, 1, 56, 56, 64, 7, 1, "f16", 5)
    S = sets(d64)
    o64 = torch.empty_like(S[0][0])

    def f64(i):
        q, k, v, rpb = S[i % len(S)]
        na.na2d_forward(q, k, v, rpb, 7, 1, out=o64)
    ms = time_calls(f64, len(S), warmup, dev)
    record("head_dim_64", d64, ms, 4 * d64.queries_heads * 128, na.na2d_last_kernel(), "D = 64")
    del S, o64

    # padded short map
    pad = Shape(128, 16, 7, 7, 32, 7, 2, "bf16", 6)
    S = sets(pad)
    op = torch.empty_like(S[0][0])

    def fpad(i):
        q, k, v, rpb = S[i % len(S)]
        na.na2d_forward(q, k, v, rpb, 7, 2, out=op)
    ms = time_calls(fpad, len(S), warmup, dev)
    record("padded_short_map", pad, ms, 4 * pad.queries_heads * 64, na.na2d_last_kernel(),
           "7x7 map with k=7, d=2: zero-padded to 14x14 and cropped")
    return out


# workloads timed beside the headline in a 1-GPU run (the second stage-1
# target first)
PER_WORKLOAD = ("dinat_s1_bf16", "dinat_sweep_bf16", "seg_bf16")


def kernels_of(wl) -> list[str]:
    """The kernel the library launched for each shape of the workload (asked
    from the library after a call, not predicted)."""
    import torch
    import neighborhood_attention_na2d_b200 as na
    names = []
    for s in wl.shapes:
        q, k, v, rpb = (t.cuda() for t in make_inputs(replace(s, B=1)))
        na.na2d_forward(q, k, v, rpb, s.k, s.d)
        names.append(na.na2d_last_kernel())
    torch.cuda.synchronize()
    return names


def run_e2e(args, wl, dev, rank, world, pg):
    import torch
    import neighborhood_attention_na2d_b200 as na

    # pinned host inputs and outputs; the library copies each step's inputs
    # in and its output back out, in chunks overlapped with the forward
    host = []
    h2d = d2h = 0
    for s in wl.shapes:
        q, k, v, rpb = make_inputs(s, s.seed + 100000 * rank)
        hq, hk, hv, hr = (t.pin_memory() for t in (q, k, v, rpb))
        hout = torch.empty_like(q).pin_memory()
        ws = torch.empty(max(1, na.na2d_forward_host_workspace_size(q.shape, s.k, s.d, q.dtype)), dtype=torch.uint8,
                         device=dev)
        host.append((s, hq, hk, hv, hr, hout, ws))
        h2d += sum(t.numel() * t.element_size() for t in (q, k, v, rpb))
        d2h += hout.numel() * hout.element_size()

    def step():
        for (s, hq, hk, hv, hr, hout, ws) in host:
            na.na2d_forward_host(hq, hk, hv, hr, s.k, s.d, out=hout, workspace=ws, device=dev)

    n = max(5, min(50, args.steps))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    stream = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    b.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), pg, dev)
    units = world * sum(s.B * s.heads * s.H * s.W for s in wl.shapes)
    return {"value": units / (ms / n / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "api": "neighborhood_attention_na2d_b200.na2d_forward_host (C ABI na2d_forward_host: "
                                "chunked host<->device copies overlapped with the forward)"}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle leg")
    ap.add_argument("--no-per-workload", action="store_true", help="time only the selected workload")
    ap.add_argument("--batch", type=int, default=None,
                    help="override B of every shape (a larger or smaller case of the same kernels)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
