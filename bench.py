"""Benchmark of the key-only GLA forward pass (libgtr.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 640|1024|2048|stack|tiny] [--path auto|split|fused]
                    [--no-sweep] [--no-cpu-baseline]

One step = one gtr_gla_fwd call over one batch of synthetic input of the
named workload (default: the 640^2 image, 40x40 grid, 1.6K tokens, 6 heads,
fp16).  Directions rotate over the workload's direction list.  Inputs and
outputs rotate over enough buffer sets that the working set exceeds the 126 MB
L2 several times, so every step streams from HBM.  The K timed steps are
captured in one CUDA graph (the pages time the operator under CUDA Graph) and
timed with CUDA events on the capture stream, bracketed by a barrier and a
device synchronise; under torchrun every rank runs its own replica and the
slowest rank's time counts.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gtr_inputs import (DTYPES, STENCILS, WORKLOADS, make_gate_epilogue_inputs, make_inputs,  # noqa: E402
                        make_lowrank_gate_inputs, make_stencil_inputs)

METRIC = "GLA fwd tokens/s and % of HBM roofline at 1.6K/4.1K/16.4K tokens, 1×B200"
L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FLOPS_PER_TOKEN_HEAD = 24704  # chunkwise, causal: 4*dk*dv + (C+1)(dk+dv)


KERNEL_SOURCES = ("gtr_fused_kernel.cuh", "gtr_sm100.cuh", "gtr_common.cuh")
TRAFFIC_DATA = os.path.join(ROOT, "profiles", "fused_gla_kernel_dram_traffic.json")


def kernel_fingerprint() -> str:
    """sha256 (first 16 hex digits) over the fused kernel's sources, in a fixed order."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "gated_token_recurrence_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """(read, write) DRAM bytes per launch that an ncu capture recorded for this workload
    (profiles/fused_gla_kernel_dram_traffic.json) -- only when the capture was taken on the
    current kernel sources (same fingerprint); (None, None) otherwise.  The write figure
    undercounts the outputs: they reach DRAM by write-back after the kernel ends."""
    try:
        with open(TRAFFIC_DATA) as f:
            rows = json.load(f)["launches"]
    except (OSError, ValueError, KeyError):
        return None, None
    fp = kernel_fingerprint()
    for row in rows:
        if row.get("workload") == workload and row.get("source") == fp:
            return int(row["dram_read_bytes"]), int(row["dram_write_bytes"])
    return None, None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        busy = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(world: int, steps: int, tokens_per_step: int, max_ms: float) -> float:
    """Whole-job throughput of `world` independent replicas: every rank processes
    `steps` x `tokens_per_step` tokens, and the job takes the slowest rank's time."""
    return world * steps * tokens_per_step / (max_ms * 1e-3)


def n_sets_for(w) -> int:
    per = w.algorithmic_bytes()
    return max(3, min(64, math.ceil(3 * L2_BYTES / per)))


def make_sets(w, n, device, rank):
    sets = []
    for i in range(n):
        d = w.direction_of_call(i)
        q, k, v, lg = make_inputs(w, w.seed(d, i) + 100000 * rank, device=device)
        out = torch.empty((w.B, w.L, w.heads, w.d_v), dtype=DTYPES[w.out_dtype], device=device)
        sets.append((d, q, k, v, lg, out))
    return sets


def time_graph(gtr, w, sets, steps, warmup, path, stream, dist, device, per_call_events=True,
               check=True):
    """Capture `steps` calls (rotating sets) in one graph; return (total_ms, per-call ms list)."""
    ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, w.d_k, w.d_v,
                           {"f32": 0, "f16": 1, "bf16": 2}[w.dtype], path, device)

    def call(i):
        d, q, k, v, lg, out = sets[i % len(sets)]
        gtr.gla_fwd(q, k, v, lg, grid=(w.H, w.W), direction=d, out=out, path=path, workspace=ws,
                    stream=stream)

    with torch.cuda.stream(stream):
        for i in range(max(warmup, 1)):
            call(i)
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)] if per_call_events else []
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            if per_call_events:
                evs[i].record(stream)
            call(i)
        if per_call_events:
            evs[steps].record(stream)
    # torch replays a graph on the CURRENT stream: make that the timed stream
    with torch.cuda.stream(stream):
        g.replay()  # warm replay
    torch.cuda.synchronize()
    if check:
        # the graph really did the work: its last output equals an eager call's, bit for bit
        i = steps - 1
        d, q, k, v, lg, out = sets[i % len(sets)]
        ref = gtr.gla_fwd(q, k, v, lg, grid=(w.H, w.W), direction=d, path=path, workspace=ws,
                          stream=stream)
        torch.cuda.synchronize()
        if not torch.equal(ref, out):
            raise RuntimeError("graph replay output differs from an eager call")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        g.replay()
        end.record(stream)
    torch.cuda.synchronize()
    barrier(dist)
    total = start.elapsed_time(end)
    per = [total / steps] * steps  # the average launch over the timed region
    if per_call_events:
        try:
            per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
        except RuntimeError:  # event nodes not timeable: keep the replay average
            pass
    del g
    return total, per


def host_cores() -> int:
    """Cores this process may run on (the oracle's OpenMP threads)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_sample(w, seconds=10.0):
    """The fp64 oracle as it stands: whole calls of the workload (every batch and head) on
    all host cores, repeated for about `seconds`, plus one whole call on one core."""
    import oracle
    d = w.directions[0]
    q, k, v, lg = make_inputs(w, w.seed(d))
    cores = host_cores()
    oracle.gla_fwd(q, k, v, lg, w.H, w.W, d, threads=cores)  # build + warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.gla_fwd(q, k, v, lg, w.H, w.W, d, threads=cores)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds or n >= 1000:
            break
    full_call_s = el / n
    t1 = time.perf_counter()
    oracle.gla_fwd(q, k, v, lg, w.H, w.W, d, threads=1)
    one_core_s = time.perf_counter() - t1
    return {"value": w.B * w.L / full_call_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "full_call_s": full_call_s, "one_core_s": one_core_s,
            "sample": f"{n} whole oracle calls of the {w.name} workload (B={w.B}, {w.heads} heads, "
                      f"L={w.L}, d_k=d_v={w.d_k}, fp64, direction {d}) on {cores} cores in {el:.1f} s, "
                      f"and one whole call on 1 core ({one_core_s:.2f} s)"}


def sweep(gtr, names, path, device, stream, hbm):
    res = {}
    for name in names:
        w = WORKLOADS[name]
        sets = make_sets(w, n_sets_for(w), device, 0)
        steps = 2 * len(sets)
        total, per = time_graph(gtr, w, sets, steps, 3, path, stream, None, device, per_call_events=False)
        mean = sum(per) / len(per)
        gbs = w.algorithmic_bytes() / (mean * 1e-3) / 1e9
        res[name] = {"L": w.L, "tokens_per_s": w.B * w.L / (mean * 1e-3),
                     "us_per_call": mean * 1e3, "GBps": gbs, "hbm_frac": gbs / hbm,
                     "path": gtr.plan(w.B, w.heads, w.H, w.W, w.d_k, w.d_v,
                                      {"f32": 0, "f16": 1, "bf16": 2}[w.dtype])[0]}
        del sets
        torch.cuda.empty_cache()
    return res


def time_rotating(call, n_sets, stream, reps=3):
    """Median per-call time (ms) of `call(i)` over rotating buffer sets i, 2 * n_sets calls
    captured in one CUDA graph and timed with one event pair on the capture stream."""
    with torch.cuda.stream(stream):
        for i in range(3):
            call(i)
    torch.cuda.synchronize()
    steps = 2 * n_sets
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            call(i)
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) / steps)
    del g
    return statistics.median(times)


def sweep_pieces(gtr, device, stream, hbm):
    """The d_k = 32 operator (the pages' kernel shape), the full GTR block call (low-rank
    gate producer + RMSNorm/SiLU output gate) and the Spatial SwiGLU stencil, each on its
    own rotating buffer sets; algorithmic bytes per call / device time per call."""
    res = {}
    code = {"f32": 0, "f16": 1, "bf16": 2}

    def line(name, bytes_, ms, tokens, extra=None):
        gbs = bytes_ / (ms * 1e-3) / 1e9
        d = {"us_per_call": ms * 1e3, "tokens_per_s": tokens / (ms * 1e-3), "GBps": gbs, "hbm_frac": gbs / hbm,
             "bytes_per_call": bytes_}
        d.update(extra or {})
        res[name] = d

    for base in ("640", "2048"):  # d_k = 32, d_v = 64
        w = WORKLOADS[base].with_(d_k=32)
        sets = make_sets(w, n_sets_for(w), device, 0)
        ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, w.d_k, w.d_v, code[w.dtype], "auto", device)

        def call(i, sets=sets, w=w, ws=ws):
            d, q, k, v, lg, out = sets[i % len(sets)]
            gtr.gla_fwd(q, k, v, lg, grid=(w.H, w.W), direction=d, out=out, workspace=ws, stream=stream)
        line(base + "_dk32", w.algorithmic_bytes(), time_rotating(call, len(sets), stream), w.B * w.L,
             {"d_k": 32, "path": gtr.plan(w.B, w.heads, w.H, w.W, 32, 64, code[w.dtype])[0]})
        del sets
        torch.cuda.empty_cache()

    # the block call at 2048^2: z (rank 16, per token) replaces the fp32 gates, the output
    # gate is read in the epilogue
    w = WORKLOADS["2048"]
    es = torch.finfo(DTYPES[w.dtype]).bits // 8
    eo = torch.finfo(DTYPES[w.out_dtype]).bits // 8
    blk_bytes = w.token_heads * ((2 * w.d_k + w.d_v) * es + w.d_v * es + w.d_v * eo) + w.B * w.L * 16 * 4
    n = max(3, min(64, math.ceil(3 * L2_BYTES / blk_bytes)))
    bsets = []
    for i in range(n):
        d = w.direction_of_call(i)
        q, k, v, _ = make_inputs(w, w.seed(d, i), device=device)
        z, w2, b = (t.to(device) for t in make_lowrank_gate_inputs(w, w.seed(d, i)))
        og, nw, eps = make_gate_epilogue_inputs(w, w.seed(d, i))
        out = torch.empty((w.B, w.L, w.heads, w.d_v), dtype=DTYPES[w.out_dtype], device=device)
        bsets.append((d, q, k, v, z, w2, b, og.to(device), nw.to(device), eps, out))
    ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, w.d_k, w.d_v, code[w.dtype], "auto", device)

    def bcall(i):
        d, q, k, v, z, w2, b, og, nw, eps, out = bsets[i % n]
        gtr.gla_block_fwd(q, k, v, grid=(w.H, w.W), direction=d, gate_z=z, gate_w2=w2, gate_b=b, gate_tau=16.0,
                          out_gate=og, norm_w=nw, norm_eps=eps, out=out, workspace=ws, stream=stream)
    line("2048_block", blk_bytes, time_rotating(bcall, n, stream), w.B * w.L, {"pieces": "lowrank gate + output gate"})
    del bsets
    torch.cuda.empty_cache()

    for name, st in STENCILS.items():  # SiLU(xg) * DWConv3x3(xv)
        n = max(3, min(64, math.ceil(3 * L2_BYTES / st.algorithmic_bytes())))
        ssets = []
        for i in range(n):
            xg, xv, cw, cb = (t.to(device) for t in make_stencil_inputs(st, 9000 + i))
            ssets.append((xg, xv, cw, cb, torch.empty_like(xv)))

        def scall(i, ssets=ssets, st=st):
            xg, xv, cw, cb, out = ssets[i % len(ssets)]
            gtr.sswiglu_dwconv(xg, xv, cw, cb, grid=(st.H, st.W), out=out, stream=stream)
        line(name, st.algorithmic_bytes(), time_rotating(scall, n, stream), st.B * st.L,
             {"C": st.C, "dtype": st.dtype})
        del ssets
        torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- arms
def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    import oracle
    d = w.directions[0]
    q, k, v, lg = make_inputs(w, w.seed(d))
    cores = host_cores()
    for _ in range(args.warmup):
        oracle.gla_fwd(q, k, v, lg, w.H, w.W, d, threads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gla_fwd(q, k, v, lg, w.H, w.W, d, threads=cores)
    el = time.perf_counter() - t0
    value = args.steps * w.B * w.L / el
    sample = (f"each step: one whole fp64 oracle call of the {w.name} workload (B={w.B}, "
              f"{w.heads} heads, L={w.L}, direction {d}) on {cores} cores")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "grid": [w.H, w.W], "heads": w.heads,
                       "d_k": w.d_k, "d_v": w.d_v, "seq_len": w.L, "in_dtype": w.dtype},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample, "full_call_s": el / args.steps},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    world, rank, local = dist_env()
    dist = init_dist(world, local)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import gated_token_recurrence_b200 as gtr

    w = WORKLOADS[args.workload]
    hbm, tc, peak_kind = peaks()
    path_name, launches = gtr.plan(w.B, w.heads, w.H, w.W, w.d_k, w.d_v,
                                   {"f32": 0, "f16": 1, "bf16": 2}[w.dtype])
    if args.path != "auto":
        path_name = args.path
    stream = torch.cuda.Stream(device)
    sets = make_sets(w, n_sets_for(w), device, rank)

    uuid = str(getattr(torch.cuda.get_device_properties(device), "uuid", ""))
    clocks = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or local))
    clocks.start()
    # soak ~1 s so the clock record covers a busy GPU, then the K timed steps
    soak_steps = 4 * len(sets)
    time_graph(gtr, w, sets, soak_steps, args.warmup, args.path, stream, None, device,
               per_call_events=False)
    # one event pair around the K graphed calls (no event nodes between the calls: consecutive
    # launches may overlap their prologue with the previous call's tail); per call = total / K
    total_ms, per = time_graph(gtr, w, sets, args.steps, args.warmup, args.path, stream, dist,
                               device, per_call_events=False)
    clk = clocks.stop()
    total_ms = max_over_ranks(dist, total_ms, device)
    tokens_per_step = w.B * w.L
    value = replica_tokens_per_s(world, args.steps, tokens_per_step, total_ms)
    mean_call = sum(per) / len(per)
    achieved = w.algorithmic_bytes() / (mean_call * 1e-3) / 1e9

    # end to end through the host-buffer entry (pinned host memory, copies inside)
    d0, q, k, v, lg, out = sets[0]
    hq, hk, hv, hg = (t.cpu().pin_memory() for t in (q, k, v, lg))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    for _ in range(2):
        gtr.gla_fwd_host(hq, hk, hv, hg, hout, grid=(w.H, w.W), direction=d0, stream=stream)
    barrier(dist)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        gtr.gla_fwd_host(hq, hk, hv, hg, hout, grid=(w.H, w.W), direction=d0, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1), device)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hg))
    d2h = hout.numel() * hout.element_size()

    extra = {}
    if rank == 0 and world == 1 and not args.no_sweep:
        extra["sweep"] = sweep(gtr, [n for n in ("640", "1024", "2048", "stack") if n != w.name],
                               args.path, device, stream, hbm)
        extra["sweep"].update(sweep_pieces(gtr, device, stream, hbm))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w, seconds=args.cpu_seconds)

    traffic = measured_traffic(w.name) if path_name == "fused" else (None, None)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "grid": [w.H, w.W], "heads": w.heads,
                       "d_k": w.d_k, "d_v": w.d_v, "seq_len": w.L, "global_batch": w.B * world,
                       "in_dtype": w.dtype, "out_dtype": w.out_dtype,
                       "directions": list(w.directions), "path": path_name,
                       "parallelism": "replicas" if world > 1 else "single",
                       "timing": "K steps in one CUDA graph, one CUDA event pair around it on the capture stream; per call = total / K",
                       "l2": f"inputs and outputs rotate over {len(sets)} buffer sets "
                             f"({len(sets) * w.algorithmic_bytes() / 2**20:.0f} MiB > L2)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm,
                         "traffic": (traffic[0] + traffic[1]) if traffic[0] is not None else None,
                         "traffic_read": traffic[0], "traffic_write": traffic[1],
                         "peak_kind": peak_kind,
                         "kernel": f"gtr_gla_fwd call ({launches} launch"
                                   f"{'es' if launches != 1 else ''}, {path_name} path)",
                         "bytes_per_call": w.algorithmic_bytes(),
                         "us_per_call": mean_call * 1e3,
                         "tensor_frac": (w.token_heads * FLOPS_PER_TOKEN_HEAD / (mean_call * 1e-3)
                                         / 1e12) / tc},
            "e2e": {"value": replica_tokens_per_s(world, e2e_steps, tokens_per_step, e2e_ms),
                    "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps * launches,
            "clocks": clk,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        line.update(extra)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_profile(args):
    """Eager calls only (no graph, sweep, e2e or CPU leg): the command ncu captures.  A
    stencil workload name (sw640, sw1024, sw2048) profiles the Spatial SwiGLU stencil."""
    import gated_token_recurrence_b200 as gtr
    device = torch.device("cuda", 0)
    if args.workload in STENCILS:
        st = STENCILS[args.workload]
        ssets = []
        for i in range(4):
            xg, xv, cw, cb = (t.to(device) for t in make_stencil_inputs(st, 9000 + i))
            ssets.append((xg, xv, cw, cb, torch.empty_like(xv)))
        for i in range(args.warmup + args.steps):
            xg, xv, cw, cb, out = ssets[i % len(ssets)]
            gtr.sswiglu_dwconv(xg, xv, cw, cb, grid=(st.H, st.W), out=out)
        torch.cuda.synchronize()
        print(json.dumps({"profile": args.workload, "calls": args.warmup + args.steps}))
        return 0
    w = WORKLOADS[args.workload]
    sets = make_sets(w, min(n_sets_for(w), 8), device, 0)
    ws = gtr.new_workspace(w.B, w.heads, w.H, w.W, w.d_k, w.d_v,
                           {"f32": 0, "f16": 1, "bf16": 2}[w.dtype], args.path, device)
    for i in range(args.warmup + args.steps):
        d, q, k, v, lg, out = sets[i % len(sets)]
        gtr.gla_fwd(q, k, v, lg, grid=(w.H, w.W), direction=d, out=out, path=args.path, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile": w.name, "calls": args.warmup + args.steps, "path": args.path}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="640", choices=sorted(WORKLOADS) + sorted(STENCILS),
                    help="GLA workload (stencil names: --profile only)")
    ap.add_argument("--path", default="auto", choices=["auto", "split", "fused", "fused_sequential"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", action="store_true",
                    help="eager calls only, for ncu captures (prints no bench line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.workload in STENCILS and not args.profile:
        ap.error("stencil workloads run under --profile only (the bench line reports them as sweep lines)")
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
