"""Benchmark of the FluxBin LUT GEMV hot path on B200.

Metric: LUT GEMV us/call and achieved HBM GB/s (fraction of the HBM peak).
Workload (N = 1): the LLaMA-2-7B-shaped 4096 x 4096 projection, batch 1,
2 global bases + 205 salient columns (5%) with 1 extra base, mu = 8,
fp16 activations with 0.5% outlier channels, fp16 output.

A step is one replay of a CUDA graph holding R fluxbin_linear calls over R
distinct resident copies of the layer (packed signs, scales, column map and
activations), R chosen so the copies total >= 3x the L2 size: every call
streams its weights from HBM.  `value` is the algorithmic bytes of all calls
(packed signs + fp16 scales + int32 column map + fp16 x + fp16 y) per second,
summed over ranks.  Multi-GPU runs are independent replicas (weak scaling).

--impl reference times the fp64 CPU oracle (all host cores) on a bounded
sample of rows of the same layer, in the same metric.
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
    """DRAM bytes per launch from the committed ncu summary of this workload,
    if it was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", f"fluxbin_lut_kernel_{workload}.txt")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m_hash = re.search(r"^kernel_source_hash:\s*(\S+)", text, re.M)
    m_tr = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not m_hash or not m_tr or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


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

def oracle_rate(spec, layer, x, rows_per_step: int, steps: int, warmup: int):
    import oracle
    rows = np.arange(min(rows_per_step, spec.M), dtype=np.int64)
    for _ in range(warmup):
        oracle.linear(layer, x, rows=rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.linear(layer, x, rows=rows)
    dt = time.perf_counter() - t0
    frac = rows.size / spec.M
    bytes_per_step = frac * algorithmic_bytes(spec, x.shape[0])
    return bytes_per_step * steps / dt / 1e9, dt, oracle.num_threads(), rows.size


def cpu_baseline(spec, layer, x, budget_s: float = 12.0):
    """The oracle on all host cores over a bounded sample: repeated full calls
    on the first 512 rows (row rebuild in fp64 + dot product), ~budget_s seconds."""
    rows = 512
    gbs, dt, cores, nrows = oracle_rate(spec, layer, x, rows, 1, 1)
    reps = max(1, int(budget_s / max(dt, 1e-3)))
    gbs, dt, cores, nrows = oracle_rate(spec, layer, x, rows, reps, 0)
    return {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 C oracle (W rows rebuilt from signs and scales, then W x) on rows 0..{nrows - 1} of "
                      f"{spec.M}, {reps} repetitions, {dt:.1f} s; GB/s counts that fraction of the call's "
                      f"algorithmic bytes",
            "us_per_call": dt / reps * spec.M / nrows * 1e6}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def build_pool(layer, spec, B, device, l2_bytes):
    import torch
    from lut_binary_basis_b200 import fluxbin, synth
    base = fluxbin.DeviceLayer.from_host(layer, device)
    per_copy = algorithmic_bytes(spec, B)
    R = max(4, int(math.ceil(3 * l2_bytes / per_copy)))
    copies, xs, ys = [], [], []
    for i in range(R):
        d = fluxbin.DeviceLayer(base.desc, base.words.clone(), base.r.clone(), base.c.clone(), base.swords.clone(),
                                base.rs.clone(), base.cs.clone(), base.idx.clone())
        copies.append(d)
        x = synth.make_x(spec, B, synth.x_key(1, 0, i, B))
        xs.append(torch.from_numpy(x).to(device))
        ys.append(torch.zeros((B, spec.M), dtype=torch.float16, device=device))
    del base
    return copies, xs, ys, R


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

    spec = synth.layer_7b_proj()
    B = 1
    layer = synth.make_layer(spec, synth.layer_key(1, 0, 0))
    x_host = synth.make_x(spec, B, synth.x_key(1, 0, 0, B))
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    copies, xs, ys, R = build_pool(layer, spec, B, device, l2)
    ws = fluxbin.new_workspace(spec.M, B, device)
    flags = fluxbin.FLAG_EARLY_WEIGHTS  # fp16 y

    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(R):  # eager warm-up (also sets kernel attributes before capture)
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(R):
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    stream.synchronize()

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
        cb = None
        if not args.no_cpu:
            cb = cpu_baseline(spec, layer, x_host)
        cub = None if args.no_cublas else cublas_reference(layer, spec, B, device, l2, args)
        clocks = sampler.summary() if sampler else None
        result = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded)",
            "config": {"workload": "llama7b_proj_4096x4096_b1", "M": spec.M, "N": spec.N, "Kb": spec.Kb,
                       "Ks": spec.Ks, "n_sal": spec.n_sal, "mu": spec.mu, "batch": B, "y": "fp16",
                       "calls_per_step": R, "l2_policy": f"rotation over {R} distinct resident copies "
                       f"({R * per_call / 2**20:.0f} MiB > 3x L2)", "parallelism": f"replicas x{world}"},
            "us_per_call": us_per_call,
            "frac_of_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
            "effective_tflops": 2.0 * spec.M * (spec.N + spec.n_sal) * B / (us_per_call * 1e-6) / 1e12,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_source": peak_kind,
                         "traffic": profiled_traffic("llama7b_proj_4096x4096_b1"),
                         "bytes_per_launch": per_call},
            "gpu_launches": R * args.steps,
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": int(x_pin.numel() * 2),
                    "d2h_bytes_per_step": int(y_pin.numel() * 2), "steps": e2e_steps},
            "cpu_baseline": cb,
            "cublas_bf16_dense_gemv": cub,
            "clocks": clocks,
        }
        if cub and cub.get("us_per_call"):
            cub["lut_speedup_vs_dense"] = cub["us_per_call"] / us_per_call
        if args.sweep:
            result["sweep"] = run_sweep(device, l2, args)
    if world > 1:
        import torch.distributed as dist
        del g, g_e2e
        dist.destroy_process_group()
    return result


def cublas_reference(layer, spec, B, device, l2, args):
    """Dense bf16 GEMV (torch.matmul) on the reconstructed W, same L2-cold rotation."""
    import torch
    W = torch.zeros((spec.M, spec.N), dtype=torch.float32, device=device)
    for k in range(spec.Kb):
        s = torch.from_numpy(layer.signs[k]).to(device).float()
        W += torch.from_numpy(layer.r[k]).to(device).float()[:, None] * s * torch.from_numpy(layer.c[k]).to(device).float()[None, :]
    idx = torch.from_numpy(layer.sal_idx.astype(np.int64)).to(device)
    for k in range(layer.sal_signs.shape[0]):
        s = torch.from_numpy(layer.sal_signs[k]).to(device).float()
        W[:, idx] += torch.from_numpy(layer.rs[k]).to(device).float()[:, None] * s * torch.from_numpy(layer.cs[k]).to(device).float()[None, :]
    Wb = W.to(torch.bfloat16)
    del W
    per = Wb.numel() * 2
    R = max(4, int(math.ceil(3 * l2 / per)))
    Ws = [Wb.clone() for _ in range(R)]
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
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    reps = 20
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    us = e0.elapsed_time(e1) * 1e3 / (reps * R)
    gb = (per + 2 * B * (spec.M + spec.N)) / (us * 1e-6) / 1e9
    return {"us_per_call": us, "GB/s_dense_bf16_bytes": gb, "copies": R,
            "lut_speedup_vs_dense": None}


def time_layer(spec, B, device, l2, wid, steps=50, path_flags=0):
    import torch
    from lut_binary_basis_b200 import fluxbin, synth
    layer = synth.make_layer(spec, synth.layer_key(wid, 0, 0))
    copies, xs, ys, R = build_pool(layer, spec, B, device, l2)
    del layer
    ws = fluxbin.new_workspace(spec.M, B, device)
    flags = fluxbin.FLAG_EARLY_WEIGHTS | path_flags
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(R):
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(R):
            copies[i].linear(xs[i], ys[i], flags, ws, stream)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    us = e0.elapsed_time(e1) * 1e3 / (steps * R)
    per = algorithmic_bytes(spec, B)
    gbs = per / (us * 1e-6) / 1e9
    peak, _ = measured_peaks()
    del g, copies, xs, ys
    torch.cuda.empty_cache()
    lk = lookups(spec, B) / (us * 1e-6)
    lds_peak = torch.cuda.get_device_properties(device).multi_processor_count * LDS_PER_CLK_PER_SM * SM_MAX_MHZ * 1e6
    return {"layer": spec.name, "B": B, "mu": spec.mu, "us_per_call": us, "GB/s": gbs, "frac_measured": gbs / peak,
            "frac_nominal": gbs / NOMINAL_HBM_GBS, "lookups_per_s": lk,
            "lookup_roofline": {"achieved": lk, "peak": lds_peak, "unit": "lookups/s", "frac": lk / lds_peak,
                                "peak_source": "SMs x 32 shared loads per clock x 1965 MHz",
                                "applies_to": "the LUT path (the tensor-core path makes no table lookups)"},
            "copies": R}


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
    __graft_entry__.build()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wid, sp = find_layer(args.layer)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    from lut_binary_basis_b200 import fluxbin
    path = {"auto": 0, "lut": fluxbin.FLAG_PATH_LUT, "tc": fluxbin.FLAG_PATH_TC}[args.path]
    return {**time_layer(sp, args.batch, device, l2, wid, steps=args.steps, path_flags=path), "path": args.path}


def run_sweep(device, l2, args):
    from lut_binary_basis_b200 import synth
    out = []
    for wid, specs, batches in ((2, synth.layers_7b_mlp(), [1, 2, 4, 8]),
                                (3, synth.layers_70b_mlp(8) + synth.layers_70b_mlp(4), [1, 16])):
        for sp in specs:
            for B in batches:
                out.append(time_layer(sp, B, device, l2, wid))
    return out


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


def run_stack(args):
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
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    layers = build_stack(device, n_layers, workers)
    setup_s = time.time() - t0
    ws = fluxbin.new_workspace(max(sp.M for sp, *_ in layers), 1, device)
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
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize(device)
    props = torch.cuda.get_device_properties(device)
    sampler = ClockSampler(gpu_id_for_smi(props)) if not args.no_clocks else None
    if sampler:
        sampler.start()
        time.sleep(0.2)
        sampler.mark(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            g.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark(False)
        sampler.stop()
    secs = e0.elapsed_time(e1) / 1e3 / args.steps
    total = sum(algorithmic_bytes(sp, 1) for sp, *_ in layers)
    peak, peak_kind = measured_peaks()
    gbs = total / secs / 1e9
    specs = synth.layers_7b_stack_linears()
    return {"metric": "LLaMA-2-7B-shaped decoder stack, linears only: decode step time (batch 1)",
            "value": secs * 1e6, "unit": "us/token", "higher_is_better": False, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "tokens_per_s": 1.0 / secs,
            "dtype": "f32", "data": "synthetic (seeded)",
            "config": {"workload": "llama7b_stack_32x7_275bit_b1", "layers": n_layers,
                       "linears": len(layers), "bits_per_weight": stack_bits_per_weight(specs),
                       "graph": "one CUDA graph, linears chained in order with programmatic dependent launch",
                       "l2_policy": f"weights {total / 2**30:.2f} GiB per step > L2"},
            "achieved_gbs": gbs, "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                                              "frac": gbs / peak, "peak_source": peak_kind},
            "gpu_launches": len(layers) * args.steps, "setup_s": setup_s,
            "clocks": sampler.summary() if sampler else None}


def run_reference(args, rank, world):
    """The oracle (CPU, all host cores) on a bounded sample of the same layer."""
    if rank != 0:
        return None
    from lut_binary_basis_b200 import synth
    import oracle
    oracle.build()
    spec = synth.layer_7b_proj()
    layer = synth.make_layer(spec, synth.layer_key(1, 0, 0))
    x = synth.make_x(spec, 1, synth.x_key(1, 0, 0, 1))
    rows_per_step = 32
    gbs, dt, cores, nrows = oracle_rate(spec, layer, x, rows_per_step, args.steps, args.warmup)
    us_per_call = dt / args.steps * spec.M / nrows * 1e6
    sample = f"fp64 C oracle on rows 0..{nrows - 1} of {spec.M} per step (row rebuild + dot), {args.steps} steps"
    return {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": "llama7b_proj_4096x4096_b1", "M": spec.M, "N": spec.N, "Kb": spec.Kb,
                       "Ks": spec.Ks, "n_sal": spec.n_sal, "mu": spec.mu, "batch": 1,
                       "parallelism": "host cores"},
            "us_per_call": us_per_call,
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": gbs, "unit": "GB/s"},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sweep", action="store_true", help="also time the 7B MLP and 70B MLP layers at their batches")
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
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    rank, local_rank, world = dist_env()
    if args.layer:
        print(json.dumps(run_one_layer(args)), flush=True)
        return
    if args.stack:
        print(json.dumps(run_stack(args)), flush=True)
        return
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_ours(args, rank, local_rank, world)
    if res is not None and rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
