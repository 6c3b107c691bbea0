"""Benchmark of the FluxBin LUT GEMV hot path on B200.

Metric: LUT GEMV us/call and achieved HBM GB/s (fraction of the HBM peak),
batch 1-16.

Headline workload (N = 1): the 70B-shaped MLP up projection 28672 x 8192,
batch 1, 2 global bases + 246 salient columns (3%) with 2 extra bases,
mu = 8, fp16 activations N(0,1) with 0.5% outlier channels x20, fp16 output
-- the largest single-layer configuration, on which the batch-1 LUT GEMV is
expected to approach the HBM roofline.  A step is one replay of a CUDA graph
holding R fluxbin_linear calls over R distinct resident copies of the layer
(packed signs, scales, column map and activations), R chosen so the copies
total >= 3x the L2 size: every call streams its weights from HBM.  `value` is
the algorithmic bytes of all calls (packed signs + fp16 scales + int32
column map + fp16 x + fp16 y) per second, summed over ranks.  Multi-GPU runs
are independent replicas (weak scaling).

The same JSON line carries, under "configs", every other configuration
timed the same way (the 4096 x 4096 projection; the 7B MLP shapes at batch
1, 2, 4, 8; the 70B MLP shapes at mu = 8 and 4, batch 1 and 16), each with
its graph-pipelined and serialised time per call, under "stack" the
32-layer 2.75-bit LLaMA-2-7B-shaped stack of linears under one CUDA graph,
and under "precompute_fusion" the batch-1 layer with its table precompute
fused into the preceding RMS normalisation against the precompute as its
own kernel and against the default path.

--impl reference times the fp64 CPU oracle (all host cores) on the bounded
sample of the headline layer that the cpu_baseline leg uses, in the same
metric.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LUT GEMV µs/call & achieved HBM GB/s (frac of ~8 TB/s peak), batch 1–16"
NOMINAL_HBM_GBS = 8000.0
# Shared-memory lookup roofline for batches >= 2 (one 4-byte table load per
# weight byte, base and batch row at mu = 8): 32 loads per clock per SM at the
# B200's maximum SM clock.
LDS_PER_CLK_PER_SM = 32
SM_MAX_MHZ = 1965.0
FALLBACK_HBM_GBS = 6650.0


# ----------------------------------------------------------------------------
# Accounting (algorithmic bytes per call)
# ----------------------------------------------------------------------------

def algorithmic_bytes(spec, B: int, y_bytes: int = 2) -> int:
    """Bytes one call must move: packed signs of both branches (unpadded),
    fp16 row and column scales, int32 salient column map, fp16 activations and
    the output."""
    M, N, Kb = spec.M, spec.N, spec.Kb
    Ks = spec.Ks if spec.n_sal else 0
    ns = spec.n_sal if Ks else 0
    bits = Kb * M * N + Ks * M * ns
    ngr = -(-N // spec.row_scale_group) if spec.row_scale_group else 1
    ngs = -(-ns // spec.sal_scale_group) if (spec.sal_scale_group and ns) else 1
    scales = 2 * (Kb * M * ngr + Ks * M * ngs) + 2 * (Kb * N + Ks * ns)
    return bits // 8 + scales + 4 * ns + 2 * B * N + y_bytes * B * M


def lookups(spec, B: int) -> int:
    Ks = spec.Ks if spec.n_sal else 0
    return B * spec.M * (spec.Kb * spec.N + Ks * spec.n_sal) // spec.mu


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lut_binary_basis_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this workload
    (profiles/<kernel>_<workload>.txt), if it was taken on the current kernel
    sources (else None)."""
    import glob
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", f"*_{workload}.txt"))):
        text = open(p).read()
        m_hash = re.search(r"^kernel_source_hash:\s*(\S+)", text, re.M)
        m_tr = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
        if m_hash and m_tr and m_hash.group(1) == kernel_source_hash():
            return float(m_tr.group(1))
    return None


# ----------------------------------------------------------------------------
# Clock sampling
# ----------------------------------------------------------------------------

def gpu_id_for_smi(props) -> str:
    """nvidia-smi -i accepts a UUID; it is independent of CUDA_VISIBLE_DEVICES."""
    u = str(getattr(props, "uuid", "") or "")
    if u and not u.startswith("GPU-"):
        u = "GPU-" + u
    return u or "0"


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for t, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 and self.t1 and self.t0 - 0.06 <= r[0] <= self.t1 + 0.06]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in use:
            for nm, v in zip(names, r[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(reasons), "samples": len(use), "in_timed_region": bool(inside)}


# ----------------------------------------------------------------------------
# Distributed helpers (replicas; the only collective is the timing reduction)
# ----------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def max_over_ranks(value: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_gbs(bytes_per_rank_per_step: float, steps: int, world: int, max_seconds: float) -> float:
    return bytes_per_rank_per_step * steps * world / max_seconds / 1e9


# ----------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ----------------------------------------------------------------------------

def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


CPU_SAMPLE_ROWS = 8192


def _median_time(fn, reps: int) -> float:
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return statistics.median(ts)


def cpu_baseline(spec, layer, x, rows: int = CPU_SAMPLE_ROWS, reps: int = 5):
    """The fp64 oracle on the host cores over a bounded sample (the first
    `rows` output rows of the layer), four ways: single-threaded and on all
    cores, each as the full call (rows of W rebuilt from signs and scales, then
    W x) and as the GEMV alone on rows rebuilt beforehand.  Medians of `reps`
    runs; per-call times and GB/s are scaled from the sample to the whole call
    (the call's algorithmic bytes).  `value` is the all-core full call."""
    import oracle
    oracle.build()
    rr = np.arange(min(rows, spec.M), dtype=np.int64)
    frac = rr.size / spec.M
    per_call = algorithmic_bytes(spec, x.shape[0])
    cores = os.cpu_count() or 1
    out = {}
    W = oracle.rebuild_rows(layer, rr)
    for name, threads in (("single_thread", 1), ("all_cores", cores)):
        oracle.set_num_threads(threads)
        oracle.linear(layer, x, rows=rr[:256])   # warm-up
        full = _median_time(lambda: oracle.linear(layer, x, rows=rr), reps)
        gemv = _median_time(lambda: oracle.gemv_rows(W, x), reps)
        out[name] = {"threads": threads, "full_call_us": full / frac * 1e6, "gemv_only_us": gemv / frac * 1e6,
                     "full_call_GB/s": per_call / (full / frac) / 1e9, "gemv_only_GB/s": per_call / (gemv / frac) / 1e9}
    oracle.set_num_threads(cores)
    del W
    return {"value": out["all_cores"]["full_call_GB/s"], "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"fp64 C oracle on output rows 0..{rr.size - 1} of {spec.M} ({spec.name}, batch "
                      f"{x.shape[0]}); median of {reps} runs each, single-threaded and on all {cores} cores, "
                      f"full call (rows of W rebuilt, then W x) and GEMV alone on rows rebuilt beforehand; "
                      f"times and GB/s scaled from the sample to the whole call",
            "us_per_call": out["all_cores"]["full_call_us"], **out}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

L2_BYTES = 126 * 2 ** 20   # B200 L2


def rotation_copies(spec, B, l2_bytes=L2_BYTES) -> int:
    """Distinct resident copies of a layer that total more than 3x the L2 size."""
    return max(4, int(math.ceil(3 * l2_bytes / algorithmic_bytes(spec, B))))


def build_pool(layer, spec, B, device, l2_bytes, wid=1):
    """R distinct resident copies of the layer (and R inputs and outputs),
    R chosen so that the copies total more than 3x the L2 size: every call of
    a rotation streams its weights from HBM."""
    import torch
    from lut_binary_basis_b200 import fluxbin, synth
    base = fluxbin.DeviceLayer.from_host(layer, device)
    R = rotation_copies(spec, B, max(l2_bytes, L2_BYTES)) if l2_bytes > 2 * L2_BYTES else rotation_copies(spec, B)
    copies, xs, ys = [base], [], []
    for i in range(R):
        if i:
            copies.append(fluxbin.DeviceLayer(base.desc, base.words.clone(), base.r.clone(), base.c.clone(),
                                              base.swords.clone(), base.rs.clone(), base.cs.clone(),
                                              base.idx.clone()))
        x = synth.make_x(spec, B, synth.x_key(wid, 0, i, B))
        xs.append(torch.from_numpy(x).to(device))
        ys.append(torch.zeros((B, spec.M), dtype=torch.float16, device=device))
    return copies, xs, ys, R


def capture_rotation(copies, xs, ys, ws, flags, stream):
    """One CUDA graph of the R calls of a rotation (after an eager run that also
    sets the kernels' attributes outside the capture)."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(len(copies)):
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(len(copies)):
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    stream.synchronize()
    return g


def time_graph(g, stream, steps: int, warmup: int = 3) -> float:
    """Seconds per replay (CUDA events on the replay stream)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            g.replay()
    e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps


def time_serialised(copies, xs, ys, ws, flags, stream, rounds: int = 3) -> float:
    """Median seconds of one call on its own: every call bracketed by two CUDA
    events, so it neither overlaps its predecessor nor is overlapped by its
    successor.  The calls are queued behind a ~20 ms device sleep so that the
    host's launch rate does not enter the timings."""
    import torch
    n = len(copies) * rounds
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    with torch.cuda.stream(stream):
        torch.cuda._sleep(40_000_000)
        for k in range(n):
            i = k % len(copies)
            ev[k][0].record(stream)
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
            ev[k][1].record(stream)
    stream.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev) / 1e3


def lds_peak(device) -> float:
    import torch
    return torch.cuda.get_device_properties(device).multi_processor_count * LDS_PER_CLK_PER_SM * SM_MAX_MHZ * 1e6


def layer_entry(spec, layer, B, device, l2, wid, steps=50, path_flags=0):
    """µs per call of one layer at one batch size on the path the library
    chooses (or the one forced): in a CUDA graph of R calls over R resident
    copies (programmatic dependent launch lets each call start streaming its
    weights while the previous one finishes), and serialised (median of single
    calls).  GB/s and fractions count the call's algorithmic bytes."""
    import torch
    from lut_binary_basis_b200 import fluxbin
    copies, xs, ys, R = build_pool(layer, spec, B, device, l2, wid)
    ws = copies[0].workspace(B)
    flags = fluxbin.FLAG_EARLY_WEIGHTS | path_flags
    stream = torch.cuda.Stream(device)
    g = capture_rotation(copies, xs, ys, ws, flags, stream)
    us = time_graph(g, stream, steps) / R * 1e6
    us_ser = time_serialised(copies, xs, ys, ws, flags, stream) * 1e6
    del g, copies, xs, ys
    torch.cuda.empty_cache()
    per = algorithmic_bytes(spec, B)
    peak, _ = measured_peaks()
    gbs = per / (us * 1e-6) / 1e9
    out = {"layer": spec.name, "M": spec.M, "N": spec.N, "Kb": spec.Kb, "Ks": spec.Ks, "n_sal": spec.n_sal,
           "mu": spec.mu, "B": B, "us_per_call": us, "GB/s": gbs, "frac_measured": gbs / peak,
           "frac_nominal": gbs / NOMINAL_HBM_GBS, "us_per_call_serialised": us_ser,
           "frac_measured_serialised": per / (us_ser * 1e-6) / 1e9 / peak, "bytes_per_call": per, "copies": R}
    if B >= 2:
        lk = lookups(spec, B) / (us * 1e-6)
        pk = lds_peak(device)
        out["lookup_roofline"] = {"achieved": lk, "peak": pk, "unit": "lookups/s", "frac": lk / pk,
                                  "peak_source": "SMs x 32 shared loads per clock x 1965 MHz",
                                  "applies_to": "the LUT path (the tensor-core path makes no table lookups)"}
    return out


def config_layers():
    """(workload id, layer spec, batches) of every benchmark configuration
    other than the smallest (parity-only) one: the 4096x4096 projection, the
    7B MLP shapes at batch 1-8, and the 70B MLP shapes at mu = 8 and 4,
    batch 1 and 16."""
    from lut_binary_basis_b200 import synth
    out = [(1, synth.layer_7b_proj(), [1])]
    out += [(2, sp, [1, 2, 4, 8]) for sp in synth.layers_7b_mlp()]
    for mu in (8, 4):
        out += [(3, sp, [1, 16]) for sp in synth.layers_70b_mlp(mu)]
    return out


def run_configs(device, l2, skip=None):
    """Every configuration's layers at their batch sizes (the library's path
    choice).  Layers of the same shape share one draw of signs and scales."""
    import dataclasses
    from lut_binary_basis_b200 import synth
    out = {}
    cache = {}
    for wid, sp, batches in config_layers():
        key = (wid, sp.M, sp.N)
        if key not in cache:
            cache.clear()
            cache[key] = synth.make_layer(sp, synth.layer_key(wid, 0, 0))
        layer = dataclasses.replace(cache[key], spec=sp)
        for B in batches:
            name = f"{sp.name}_b{B}"
            if skip and name in skip:
                out[name] = skip[name]
                continue
            out[name] = layer_entry(sp, layer, B, device, l2, wid)
    return out


def precompute_fusion_entry(spec, layer, device, wid, steps=50):
    """Batch 1: the layer with its table precompute fused into the preceding
    RMS normalisation (fluxbin_linear_rmsnorm, reading the un-normalised row),
    against the precompute as its own kernel on an already normalised row
    (FLUXBIN_FLAG_SEPARATE_TABLES) and against the library's default path;
    µs per call in a CUDA graph of R dependent calls over R copies (L2-cold
    like the other entries)."""
    import numpy as np
    import torch
    from lut_binary_basis_b200 import fluxbin
    copies, xs, ys, R = build_pool(layer, spec, 1, device, L2_BYTES, wid)
    ws = copies[0].workspace(1)
    gamma = torch.from_numpy(np.random.default_rng([wid, 77]).uniform(0.5, 1.5, spec.N).astype(np.float16)).to(device)
    stream = torch.cuda.Stream(device)
    ew = fluxbin.FLAG_EARLY_WEIGHTS
    calls = {
        "fused_rmsnorm_us": lambda i: copies[i].linear_rmsnorm(xs[i][0], gamma, 1e-5, ys[i], ew, ws, None, stream),
        "separate_tables_us": lambda i: copies[i].linear(xs[i], ys[i], ew | fluxbin.FLAG_SEPARATE_TABLES, ws, stream),
        "default_path_us": lambda i: copies[i].linear(xs[i], ys[i], ew, ws, stream),
    }
    out = {"layer": spec.name, "B": 1, "copies": R}
    for name, fn in calls.items():
        with torch.cuda.stream(stream):
            for i in range(R):
                fn(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(R):
                fn(i)
        out[name] = time_graph(g, stream, steps) / R * 1e6
        del g
    del copies, xs, ys
    torch.cuda.empty_cache()
    return out


def run_precompute_fusion(device):
    from lut_binary_basis_b200 import synth
    out = {}
    for wid, sp in ((HEADLINE_WID, headline_spec()), (1, synth.layer_7b_proj())):
        layer = synth.make_layer(sp, synth.layer_key(wid, 0, 0))
        out[sp.name] = precompute_fusion_entry(sp, layer, device, wid)
    return out


HEADLINE_WID = 3


def headline_spec():
    from lut_binary_basis_b200 import synth
    return synth.layers_70b_mlp(8)[0]


def workload_config(spec, B, world):
    """The `config` of the JSON line (identical in both arms)."""
    R = rotation_copies(spec, B)
    per_call = algorithmic_bytes(spec, B)
    return {"workload": f"{spec.name}_b{B}", "M": spec.M, "N": spec.N, "Kb": spec.Kb, "Ks": spec.Ks,
            "n_sal": spec.n_sal, "mu": spec.mu, "batch": B, "y": "fp16", "parallelism": f"replicas x{world}",
            "calls_per_step": R,
            "l2_policy": (f"inputs larger than L2: rotation over {R} distinct resident copies "
                          f"({R * per_call / 2**20:.0f} MiB > 3x L2)")}


def run_ours(args, rank, local_rank, world):
    import torch
    from lut_binary_basis_b200 import fluxbin, synth
    import __graft_entry__
    __graft_entry__.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)

    spec = headline_spec()
    B = 1
    layer = synth.make_layer(spec, synth.layer_key(HEADLINE_WID, 0, 0))
    x_host = synth.make_x(spec, B, synth.x_key(HEADLINE_WID, 0, 0, B))
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    copies, xs, ys, R = build_pool(layer, spec, B, device, l2, HEADLINE_WID)
    ws = copies[0].workspace(B)
    flags = fluxbin.FLAG_EARLY_WEIGHTS  # fp16 y

    stream = torch.cuda.Stream(device)
    g = capture_rotation(copies, xs, ys, ws, flags, stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize(device)

    sampler = ClockSampler(gpu_id_for_smi(props)) if not args.no_clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.2)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark(True)
    ev0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            g.replay()
    ev1.record(stream)
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark(False)
    barrier(device)
    if sampler:
        sampler.stop()
    secs = ev0.elapsed_time(ev1) / 1e3
    max_secs = max_over_ranks(secs, device)

    per_call = algorithmic_bytes(spec, B)
    value = whole_job_gbs(per_call * R, args.steps, world, max_secs)
    us_per_call = max_secs / (args.steps * R) * 1e6
    achieved = per_call / (us_per_call * 1e-6) / 1e9
    peak, peak_kind = measured_peaks()
    us_ser = time_serialised(copies, xs, ys, ws, flags, stream) * 1e6

    # end to end through the public API with host buffers: pinned x -> device,
    # the R calls, device y -> pinned host, every step (the step is captured
    # in a CUDA graph like the device-timed one, so both copies run on every
    # replay and host launch overhead is not what is measured)
    x_pin = torch.empty((R, B, spec.N), dtype=torch.float16).pin_memory()
    y_pin = torch.empty((R, B, spec.M), dtype=torch.float16).pin_memory()
    for i in range(R):
        x_pin[i].copy_(xs[i].cpu())
    x_dev = torch.empty((R, B, spec.N), dtype=torch.float16, device=device)
    y_dev = torch.empty((R, B, spec.M), dtype=torch.float16, device=device)
    e2e_steps = max(3, min(args.steps, 200))

    def e2e_step():
        x_dev.copy_(x_pin, non_blocking=True)
        for i in range(R):
            copies[i].linear(x_dev[i], y_dev[i], flags, ws, stream)
        y_pin.copy_(y_dev, non_blocking=True)

    with torch.cuda.stream(stream):
        e2e_step()
    stream.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        e2e_step()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            g_e2e.replay()
    stream.synchronize()
    barrier(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(e2e_steps):
            g_e2e.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_secs = max_over_ranks(e0.elapsed_time(e1) / 1e3, device)
    e2e_value = whole_job_gbs(per_call * R, e2e_steps, world, e2e_secs)

    result = None
    if rank == 0:
        clocks = sampler.summary() if sampler else None
        del g, g_e2e, copies, xs, ys, x_dev, y_dev
        torch.cuda.empty_cache()
        cb = None if args.no_cpu else cpu_baseline(spec, layer, x_host)
        cub = None if args.no_cublas else cublas_reference(layer, spec, B, device, l2, args)
        headline_name = f"{spec.name}_b{B}"
        headline_entry = {"layer": spec.name, "M": spec.M, "N": spec.N, "Kb": spec.Kb, "Ks": spec.Ks,
                          "n_sal": spec.n_sal, "mu": spec.mu, "B": B, "us_per_call": us_per_call,
                          "GB/s": achieved, "frac_measured": achieved / peak,
                          "frac_nominal": achieved / NOMINAL_HBM_GBS, "us_per_call_serialised": us_ser,
                          "frac_measured_serialised": per_call / (us_ser * 1e-6) / 1e9 / peak,
                          "bytes_per_call": per_call, "copies": R}
        del layer
        configs = None
        if not args.headline_only:
            configs = run_configs(device, l2, skip={headline_name: headline_entry})
        stack = None if (args.headline_only or args.no_stack) else run_stack(args, device, summary=True)
        fusion = None if args.headline_only else run_precompute_fusion(device)
        result = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
            "config": workload_config(spec, B, world),
            "us_per_call": us_per_call,
            "us_per_call_serialised": us_ser,
            "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
            "effective_tflops": 2.0 * spec.M * (spec.N + spec.n_sal) * B / (us_per_call * 1e-6) / 1e12,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": f"{peak_kind} (HBM copy bandwidth)",
                         "traffic": profiled_traffic(headline_name), "bytes_per_launch": per_call,
                         "frac_serialised": per_call / (us_ser * 1e-6) / 1e9 / peak},
            "gpu_launches": R * args.steps,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": int(x_pin.numel() * 2),
                    "d2h_bytes_per_step": int(y_pin.numel() * 2), "steps": e2e_steps},
            "cpu_baseline": cb,
            "cublas_bf16_dense_gemv": cub,
            "clocks": clocks,
            "configs": configs,
            "stack": stack,
            "precompute_fusion": fusion,
        }
        if cub and cub.get("us_per_call"):
            cub["lut_speedup_vs_dense"] = cub["us_per_call"] / us_per_call
    else:
        del g, g_e2e
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return result


def cublas_reference(layer, spec, B, device, l2, args):
    """Dense bf16 GEMV (torch.matmul) on the reconstructed W, same L2-cold rotation."""
    import torch
    W = torch.zeros((spec.M, spec.N), dtype=torch.float32, device=device)
    for k in range(spec.Kb):
        s = torch.from_numpy(layer.signs[k]).to(device).float()
        W += torch.from_numpy(layer.r[k]).to(device).float()[:, None] * s * torch.from_numpy(layer.c[k]).to(device).float()[None, :]
        del s
    idx = torch.from_numpy(layer.sal_idx.astype(np.int64)).to(device)
    for k in range(layer.sal_signs.shape[0]):
        s = torch.from_numpy(layer.sal_signs[k]).to(device).float()
        W[:, idx] += torch.from_numpy(layer.rs[k]).to(device).float()[:, None] * s * torch.from_numpy(layer.cs[k]).to(device).float()[None, :]
    Wb = W.to(torch.bfloat16)
    del W
    per = Wb.numel() * 2
    R = max(4, int(math.ceil(3 * l2 / per)))
    Ws = [Wb] + [Wb.clone() for _ in range(R - 1)]
    x = torch.randn((spec.N, B), dtype=torch.bfloat16, device=device)
    ys = [torch.empty((spec.M, B), dtype=torch.bfloat16, device=device) for _ in range(R)]
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(R):
            torch.matmul(Ws[i], x, out=ys[i])
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(R):
            torch.matmul(Ws[i], x, out=ys[i])
    secs = time_graph(g, stream, 20)
    us = secs * 1e6 / R
    gb = (per + 2 * B * (spec.M + spec.N)) / (us * 1e-6) / 1e9
    del g, Ws, ys, Wb
    torch.cuda.empty_cache()
    return {"us_per_call": us, "GB/s_dense_bf16_bytes": gb, "copies": R, "layer": spec.name, "B": B,
            "lut_speedup_vs_dense": None}


def find_layer(name):
    from lut_binary_basis_b200 import synth
    for wid, (_, specs, _) in synth.WORKLOADS.items():
        for sp in specs:
            if sp.name == name:
                return wid, sp
    raise SystemExit(f"unknown layer {name!r}")


def run_one_layer(args):
    """One layer of the workloads at one batch size (also the profiling driver)."""
    import torch
    import __graft_entry__
    from lut_binary_basis_b200 import fluxbin, synth
    __graft_entry__.build()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wid, sp = find_layer(args.layer)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    path = {"auto": 0, "lut": fluxbin.FLAG_PATH_LUT, "tc": fluxbin.FLAG_PATH_TC}[args.path]
    layer = synth.make_layer(sp, synth.layer_key(wid, 0, 0))
    return {**layer_entry(sp, layer, args.batch, device, l2, wid, steps=args.steps, path_flags=path),
            "path": args.path}


# ----------------------------------------------------------------------------
# The LLaMA-2-7B-shaped decoder stack (32 x q,k,v,o,gate,up,down), 2.75 bits
# ----------------------------------------------------------------------------

def _stack_job(job):
    """Worker: draw and pack one linear of the stack (host only)."""
    l, li = job
    from lut_binary_basis_b200 import fluxbin, synth
    sp = synth.layers_7b_stack_linears()[li]
    host = synth.make_layer(sp, synth.layer_key(4, l, li))
    packed = fluxbin.pack_host(host)
    x = synth.make_x(sp, 1, synth.x_key(4, l, li, 1))
    return l, li, packed, x


def build_stack(device, n_layers, workers):
    """Every linear of the stack resident on the device, with its own seeded
    fp16 N(0,1) input and fp16 output (the linears are chained in order but do
    not feed one another: without the normalisation and attention between
    them the outputs would overflow fp16)."""
    import multiprocessing as mp
    import torch
    from lut_binary_basis_b200 import fluxbin, synth
    specs = synth.layers_7b_stack_linears()
    jobs = [(l, li) for l in range(n_layers) for li in range(len(specs))]
    out = []
    with mp.get_context("spawn").Pool(workers) as pool:
        for l, li, packed, x in pool.imap(_stack_job, jobs, chunksize=1):
            sp = specs[li]
            out.append((sp, fluxbin.DeviceLayer.from_packed(packed, device), torch.from_numpy(x).to(device),
                        torch.empty((1, sp.M), dtype=torch.float16, device=device)))
    return out


def stack_bits_per_weight(specs) -> float:
    """Packed bits + fp16 scales + int32 column map per weight of the stack's linears."""
    bits = w = 0
    for sp in specs:
        bits += 8 * (algorithmic_bytes(sp, 1) - 2 * sp.N - 2 * sp.M)
        w += sp.M * sp.N
    return bits / w


def run_stack(args, device=None, summary=False):
    """One decode step (batch 1) through all 224 linears, chained in order
    under one CUDA graph; a step's inputs are resident and the weights (2.2 GB)
    are far larger than L2."""
    import torch
    import __graft_entry__
    from lut_binary_basis_b200 import fluxbin, synth
    __graft_entry__.build()
    n_layers = args.stack_layers
    workers = max(1, min(8, (os.cpu_count() or 2) - 1))
    t0 = time.time()
    if device is None:
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
    layers = build_stack(device, n_layers, workers)
    setup_s = time.time() - t0
    ws = max((dl.workspace(1) for _, dl, _, _ in layers), key=lambda t: t.numel())
    flags = fluxbin.FLAG_EARLY_WEIGHTS
    stream = torch.cuda.Stream(device)

    def step():
        for sp, dl, x, y in layers:
            dl.linear(x, y, flags, ws, stream)

    with torch.cuda.stream(stream):
        step()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    steps = args.stack_steps if summary else args.steps
    sampler = None
    if not summary and not args.no_clocks:
        sampler = ClockSampler(gpu_id_for_smi(torch.cuda.get_device_properties(device)))
        sampler.start()
        time.sleep(0.2)
        sampler.mark(True)
    secs = time_graph(g, stream, steps, warmup=max(3, args.warmup if not summary else 3))
    if sampler:
        sampler.mark(False)
        sampler.stop()
    total = sum(algorithmic_bytes(sp, 1) for sp, *_ in layers)
    n_linears = len(layers)
    del g, layers
    torch.cuda.empty_cache()
    peak, peak_kind = measured_peaks()
    gbs = total / secs / 1e9
    specs = synth.layers_7b_stack_linears()
    res = {"metric": "LLaMA-2-7B-shaped decoder stack, linears only: decode step time (batch 1)",
           "value": secs * 1e6, "unit": "us/token", "higher_is_better": False, "n_gpus": 1,
           "steps": steps, "tokens_per_s": 1.0 / secs, "dtype": "f32", "data": "synthetic (seeded)",
           "config": {"workload": "llama7b_stack_32x7_275bit_b1", "layers": n_layers,
                      "linears": n_linears, "bits_per_weight": stack_bits_per_weight(specs),
                      "graph": "one CUDA graph, linears chained in order with programmatic dependent launch",
                      "l2_policy": f"weights {total / 2**30:.2f} GiB per step > L2"},
           "achieved_gbs": gbs, "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                                             "frac": gbs / peak, "peak_source": peak_kind},
           "gpu_launches_per_step": n_linears, "setup_s": setup_s}
    if not summary:
        res.update({"warmup": args.warmup, "gpu_launches": n_linears * steps,
                    "clocks": sampler.summary() if sampler else None})
    return res


def run_fit(args):
    """Host decomposition fitting of a dense 4096 x 4096 matrix into the
    2.75-bit stack layout (2 global bases with G = 128 row-scale blocks, 16
    salient columns per 128-column block with 2 extra bases and one salient
    row scale per 16 of them): the library's threaded C++ fitter against the
    fp64 numpy oracle, same steps and iteration count.  W_ij = a_i b_j z_ij with
    a, b ~ LogNormal(0, 0.5), z ~ N(0, 1), seeded."""
    from lut_binary_basis_b200 import fluxbin
    from oracle import fit as ofit
    M = N = args.fit_size
    g = np.random.default_rng(2024)
    W = np.exp(0.5 * g.standard_normal(M))[:, None] * np.exp(0.5 * g.standard_normal(N))[None, :] * \
        g.standard_normal((M, N))
    S = np.concatenate([blk * 128 + np.sort(g.choice(128, 16, replace=False)) for blk in range(N // 128)])
    S = S.astype(np.int32)
    it = args.fit_iters
    t0 = time.perf_counter()
    res = fluxbin.fluxbin_fit_hybrid(W, 2, S, 2, 128, 16, it)
    t_lib = time.perf_counter() - t0
    out = {"metric": "host decomposition fitting time", "unit": "s", "M": M, "N": N, "Kb": 2, "G": 128, "Ks": 2,
           "n_sal": int(S.size), "Gs": 16, "iters": it, "threads": os.cpu_count(), "cpu_model": cpu_model(),
           "library_s": t_lib, "relative_error": math.sqrt(res[-1] / float(np.sum(W * W)))}
    if not args.no_cpu:
        t0 = time.perf_counter()
        (gs, gr, gc), (ss, sr, sc) = ofit.fit_hybrid(W, S, 2, 2, 128, 16, it)
        out["oracle_s"] = time.perf_counter() - t0
        out["signs_equal"] = bool(np.array_equal(gs, res[0]) and np.array_equal(ss, res[3]))
    return out


def run_reference(args, rank, world):
    """The oracle (CPU, all host cores): every step is one full call (rows of W
    rebuilt from signs and scales, then W x) on the same bounded sample of the
    benchmark's layer that the cpu_baseline leg times."""
    if rank != 0:
        return None
    from lut_binary_basis_b200 import synth
    import oracle
    oracle.build()
    spec = headline_spec()
    layer = synth.make_layer(spec, synth.layer_key(HEADLINE_WID, 0, 0))
    x = synth.make_x(spec, 1, synth.x_key(HEADLINE_WID, 0, 0, 1))
    rr = np.arange(min(CPU_SAMPLE_ROWS, spec.M), dtype=np.int64)
    frac = rr.size / spec.M
    for _ in range(args.warmup):
        oracle.linear(layer, x, rows=rr)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear(layer, x, rows=rr)
    dt = time.perf_counter() - t0
    per_call = algorithmic_bytes(spec, 1)
    gbs = frac * per_call * args.steps / dt / 1e9 if dt > 0 else 0.0
    cores = oracle.num_threads()
    sample = (f"fp64 C oracle on all {cores} host cores ({cpu_model()}): output rows 0..{rr.size - 1} of "
              f"{spec.M} per step (rows of W rebuilt, then W x), {args.steps} steps; GB/s counts that "
              f"fraction of the call's algorithmic bytes")
    cfg = workload_config(spec, 1, world)
    return {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / max(args.steps, 1) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": cfg,
            "us_per_call": dt / max(args.steps, 1) / frac * 1e6,
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": gbs, "unit": "GB/s"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline layer (no other configurations, no stack)")
    ap.add_argument("--no-stack", action="store_true", help="skip the decoder-stack entry")
    ap.add_argument("--stack-steps", type=int, default=20, help="graph replays timed for the stack entry")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-cublas", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--layer", default=None,
                    help="time one named layer of the workloads instead (e.g. llama7b_gate_up_11008x4096)")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--path", choices=("auto", "lut", "tc"), default="auto",
                    help="with --layer: force the LUT or the tensor-core path (default: the library's choice)")
    ap.add_argument("--stack", action="store_true",
                    help="time the 32-layer LLaMA-2-7B-shaped stack of 2.75-bit linears instead")
    ap.add_argument("--stack-layers", type=int, default=32)
    ap.add_argument("--fit", action="store_true",
                    help="time the host decomposition fitter (library vs oracle) on a dense matrix instead")
    ap.add_argument("--fit-size", type=int, default=4096)
    ap.add_argument("--fit-iters", type=int, default=5)
    ap.add_argument("--fusion", action="store_true",
                    help="time the headline layer with its table precompute fused into the preceding RMS "
                         "normalisation, against the precompute on a normalised row and the default path, instead")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    rank, local_rank, world = dist_env()
    if args.layer:
        print(json.dumps(run_one_layer(args)), flush=True)
        return
    if args.stack:
        print(json.dumps(run_stack(args)), flush=True)
        return
    if args.fit:
        print(json.dumps(run_fit(args)), flush=True)
        return
    if args.fusion:
        import torch
        import __graft_entry__
        from lut_binary_basis_b200 import synth
        __graft_entry__.build()
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        sp = headline_spec()
        layer = synth.make_layer(sp, synth.layer_key(HEADLINE_WID, 0, 0))
        print(json.dumps(precompute_fusion_entry(sp, layer, device, HEADLINE_WID, steps=args.steps)), flush=True)
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, local_rank, world)
    if res is not None and rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
