#!/usr/bin/env python3
"""Throughput of the TTQ hot path: prompt tokens/s per layer, including the
on-the-fly quantization.

One step is one pass of the whole path over one prompt of the workload: for
every distinct layer input, statistics and scales (one launch) -> prepared
fp16 operand; for every layer, group RTN of its weight -> tensor-core
low-bit projection. Layers that share an input run as one projection of
their stacked weights, and the prepared operand is built on a second stream
while the weights are quantized. The default workload is an OPT-125M-shaped
block (q, k, v, o 768x768, fc1 3072x768, fc2 768x3072; q, k, v share one
input), T = 2048, b = 3, g = 32.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs an independent replica
(the path has no exchange step), the timed region is bracketed by a barrier
and a device synchronisation, and the slowest rank's time counts.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs  # noqa

METRIC = "prompt tokens/s per layer incl. on-the-fly quant"
L2_BYTES = 126 * 1024 * 1024
ORACLE_SAMPLE_TOKENS = 128
REFERENCE_SECONDS = 60.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 5000 steps of ~0.13 ms keep the GPU busy for ~0.6 s, long enough for
    # several clock samples inside the timed region
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="opt125m-block",
                    choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the step directly instead of replaying a "
                         "CUDA graph (for profilers)")
    ap.add_argument("--separate", action="store_true",
                    help="one call per step of the method and per layer, on "
                         "one stream (no fused launches, for comparison)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained",
                                               d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------ workload ----

def layer_inputs(wl):
    """Distinct layer inputs in the order the layers first use them."""
    out = []
    for L in wl.layers:
        if L.input_name not in out:
            out.append(L.input_name)
    return out


def projection_groups(wl, separate=False):
    """(name, input name, layers): layers that share an input and carry no
    low-rank factors of their own run as one projection."""
    groups = []
    for k in layer_inputs(wl):
        Ls = [L for L in wl.layers if L.input_name == k]
        if separate or wl.rank or len(Ls) == 1:
            groups += [(L.name, k, [L]) for L in Ls]
        else:
            groups.append(("|".join(L.name for L in Ls), k, Ls))
    return groups


def launch_plan(inputs, groups, separate=False):
    """(kind, key) of every call of one step, in launch order."""
    plan = []
    for k in inputs:
        plan += [("stats", k), ("scales", k)] if separate else \
            [("stats_scales", k)]
        plan.append(("prepare", k))
        mine = [g for g, kk, _ in groups if kk == k]
        plan += [("quantize", g) for g in mine]
        plan += [("gemm", g) for g in mine]
    return plan


class Step:
    """Device buffers and the launch sequence of one step.

    Layers that share an input (q, k, v) run as one projection whose weight
    is the layers' rows stacked ([2304, 768] for q|k|v): group RTN works row
    by row and the projection column by column, so every code and output is
    the one the separate layers would give. Per input the order is the
    method's: statistics and scales (one launch) -> the prepared operand on
    a second stream, beside the quantization of the weights on the first ->
    the projections. ``separate`` restores one call per step of the method
    and per layer on a single stream (for comparison)."""

    def __init__(self, ttq, wl, data, device, replicas, separate=False):
        self.ttq, self.wl = ttq, wl
        self.T = wl.T
        self.separate = separate
        self.inputs = layer_inputs(wl)
        self.groups = projection_groups(wl, separate)
        self.R = replicas
        self.X = [{k: v.to(device) for k, v in data["X"].items()}
                  for _ in range(replicas)]
        self.W = []
        for _ in range(replicas):
            self.W.append({g: torch.cat([data["W"][L.name] for L in Ls]).to(
                device).contiguous() for g, _, Ls in self.groups})
        self.A = {k: v.to(device) for k, v in data["A"].items()}
        self.B = {k: v.to(device) for k, v in data["B"].items()}
        f32 = dict(dtype=torch.float32, device=device)
        self.sums = {k: torch.empty(self.X[0][k].shape[1], **f32)
                     for k in self.inputs}
        self.s = {k: torch.empty_like(v) for k, v in self.sums.items()}
        self.inv = {k: torch.empty_like(v) for k, v in self.sums.items()}
        self.counter = ttq.new_counter(device)
        self.Xs = {k: torch.empty(self.X[0][k].shape, dtype=torch.float16,
                                  device=device) for k in self.inputs}
        r = wl.rank
        self.U = {k: torch.empty((self.T, 64), dtype=torch.float16,
                                 device=device) for k in self.inputs} if r \
            else {}
        b, g = wl.bits, wl.group
        self.codes, self.delta, self.zero, self.Y, self.N = {}, {}, {}, {}, {}
        for name, _, Ls in self.groups:
            N, K = sum(L.N for L in Ls), Ls[0].K
            self.N[name] = N
            self.codes[name] = torch.empty((N, ttq.codes_ld(K, b)),
                                           dtype=torch.int32, device=device)
            gl = ttq.groups_ld(K, g)
            self.delta[name] = torch.empty((N, gl), **f32)
            self.zero[name] = torch.empty((N, gl), dtype=torch.uint8,
                                          device=device)
            self.Y[name] = torch.empty((self.T, N), dtype=wl.dtype,
                                       device=device)
        self.side = None if separate else torch.cuda.Stream(device)
        self.plan = launch_plan(self.inputs, self.groups, separate)

    def input_bytes(self):
        return sum(v.numel() * v.element_size() for v in self.X[0].values()) + \
            sum(v.numel() * v.element_size() for v in self.W[0].values())

    def kernel_launches(self):
        """Kernels one step launches (the prepare of a low-rank input runs a
        second kernel for X A^T)."""
        return len(self.plan) + (len(self.inputs) if self.wl.rank else 0)

    def _fn(self, rep, kind, key):
        t, wl = self.ttq, self.wl
        X, W = self.X[rep], self.W[rep]
        if kind == "stats":
            return lambda: t.act_stats(X[key], wl.p, out=self.sums[key])
        if kind == "scales":
            return lambda: t.awq_scales(self.sums[key], self.T, wl.alpha,
                                        wl.lam, wl.p, self.s[key],
                                        self.inv[key])
        if kind == "stats_scales":
            return lambda: t.act_stats_scales(
                X[key], self.counter, wl.alpha, wl.lam, wl.p, self.sums[key],
                self.s[key], self.inv[key])
        if kind == "prepare":
            A = None
            if wl.rank:
                # the low-rank factors belong to a layer; layers that share
                # an input in these workloads never both carry factors
                owner = next(g for g, k, _ in self.groups if k == key)
                A = self.A[owner]
            return lambda: t.prepare_activations(
                X[key], self.inv[key], wl.bits, A, self.Xs[key],
                self.U.get(key))
        k = next(kk for g, kk, _ in self.groups if g == key)
        if kind == "quantize":
            return lambda: t.quantize_rtn_grouped(
                W[key], self.s[k], wl.bits, wl.group, self.codes[key],
                self.delta[key], self.zero[key])
        return lambda: t.w_lowbit_gemm_prepared(
            self.Xs[k], self.U.get(k), self.codes[key], self.delta[key],
            self.zero[key], self.N[key], wl.bits, wl.group,
            self.B.get(key) if wl.rank else None, out=self.Y[key])

    def run(self, rep, events=None):
        main = torch.cuda.current_stream()
        joins = {}
        for i, (kind, key) in enumerate(self.plan):
            fn = self._fn(rep, kind, key)
            on_side = kind == "prepare" and self.side is not None
            if kind == "gemm" and key in joins:
                main.wait_event(joins.pop(key))
            if on_side:
                fork = torch.cuda.Event()
                fork.record(main)
                self.side.wait_event(fork)
            st = self.side if on_side else main
            with torch.cuda.stream(st):
                if events is not None:
                    events[i][0].record()
                fn()
                if events is not None:
                    events[i][1].record()
            if on_side:
                done = torch.cuda.Event()
                done.record(self.side)
                for g, kk, _ in self.groups:
                    if kk == key:
                        joins[g] = done


def algorithmic_work(wl):
    """Bytes (HBM-bound steps) and flops (projection) per step, from the
    algorithmic minimum: every input read once, every output written once."""
    T, b, g = wl.T, wl.bits, wl.group
    xb = 2 if wl.dtype != torch.float32 else 4
    seen, w = set(), {"stats": 0, "scales": 0, "prepare": 0, "quantize": 0,
                      "gemm": 0, "gemm_flops": 0}
    # (the fused statistics + scales launch moves both steps' bytes)
    for L in wl.layers:
        if L.input_name not in seen:
            seen.add(L.input_name)
            w["stats"] += T * L.K * xb + L.K * 4
            w["scales"] += L.K * 12
            w["prepare"] += T * L.K * (xb + 2) + L.K * 4
        w["quantize"] += L.N * L.K * xb + L.K * 4 + L.N * L.K * b // 8 + \
            5 * L.N * L.K // g
        w["gemm"] += T * L.K * 2 + L.N * L.K * b // 8 + 5 * L.N * L.K // g + \
            T * L.N * xb
        w["gemm_flops"] += 2 * T * L.N * L.K + 2 * T * wl.rank * (L.K + L.N)
    w["stats_scales"] = w["stats"] + w["scales"]
    return w


# -------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi samples every 100 ms; the summary keeps the samples taken
    between mark_start() and mark_end() (all of them, flagged, if none
    fell inside)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = datetime.datetime.now()

    def mark_end(self):
        self.t1 = datetime.datetime.now()

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.summarize(lines, self.t0, self.t1)

    @staticmethod
    def summarize(lines, t0=None, t1=None):
        """Median SM clock, max clock and active throttle reasons of the CSV
        rows (timestamp first) that fall in [t0, t1]."""
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0],
                                                "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(parts[2]), float(parts[3]),
                             parts[6:10]))
            except ValueError:
                continue
        if not rows:
            return None
        inside = rows
        if t0 is not None and t1 is not None:
            slack = datetime.timedelta(milliseconds=50)
            inside = [r for r in rows if r[0] is not None and
                      t0 - slack <= r[0] <= t1 + slack]
        in_region = bool(inside)
        use = inside if inside else rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for *_, r in use for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use), "samples": len(use),
                "in_timed_region": in_region, "reasons": reasons}


# ------------------------------------------------------------- oracle -----

def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _ranges(n, parts):
    """[lo, hi) pieces of range(n), at most ``parts`` of near-equal size."""
    parts = max(1, min(parts, n))
    b = [n * i // parts for i in range(parts + 1)]
    return [(b[i], b[i + 1]) for i in range(parts)]


def oracle_step(wl, data, sample_tokens, threads=1, outputs=None):
    """The CPU oracle on a bounded sample of one step: statistics, scales and
    quantization at full size, the projection on the first ``sample_tokens``
    tokens, scaled linearly to T. Returns (seconds per step, description).

    With ``threads`` > 1 the unchanged oracle functions run concurrently on
    disjoint slices: the statistics over token ranges (the partial sums are
    added), the quantizer and the projection over output rows. The C calls
    release the GIL. ``outputs``, when a dict, receives every layer's
    (codes, delta, zero, Y sample) for checking."""
    import numpy as np
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    T = wl.T
    Ts = min(sample_tokens, T)
    Xn = {k: v.float().numpy() for k, v in data["X"].items()}
    pool = ThreadPoolExecutor(threads) if threads > 1 else None

    def each(fn, n):
        pieces = _ranges(n, threads)
        if pool is None:
            return [fn(a, b) for a, b in pieces]
        return list(pool.map(lambda ab: fn(*ab), pieces))

    try:
        t0 = time.perf_counter()
        s, inv = {}, {}
        for k, X in Xn.items():
            sums = sum(each(lambda a, b: oracle.act_sums(X[a:b], wl.p), T))
            s[k], inv[k] = oracle.awq_scales(sums, T, wl.alpha, wl.lam, wl.p)
        t_full = time.perf_counter() - t0
        t_gemm = 0.0
        for L in wl.layers:
            W = data["W"][L.name].float().numpy()
            s32 = s[L.input_name].astype(np.float32)
            t1 = time.perf_counter()
            parts = each(lambda a, b: oracle.quantize(W[a:b], s32, wl.bits,
                                                      wl.group), L.N)
            c, d, z = (np.concatenate(x) for x in zip(*parts))
            t_full += time.perf_counter() - t1
            A = B = None
            if wl.rank:
                A = data["A"][L.name].float().numpy()
                B = data["B"][L.name].float().numpy()
            Xs = Xn[L.input_name][:Ts]
            t2 = time.perf_counter()
            ys = each(lambda a, b: oracle.lowbit_gemm(
                Xs, inv[L.input_name], c[a:b], d[a:b], z[a:b], b - a, wl.bits,
                wl.group, A, None if B is None else B[a:b]), L.N)
            t_gemm += time.perf_counter() - t2
            if outputs is not None:
                outputs[L.name] = (c, d, z, np.concatenate(ys, axis=1))
    finally:
        if pool is not None:
            pool.shutdown()
    est = t_full + t_gemm * (T / Ts)
    how = ("1 thread" if threads == 1 else
           f"{threads} threads on disjoint token ranges (statistics) and "
           f"output rows (quantizer, projection)")
    desc = (f"stats, scales and quantize at full size; projection on {Ts} of "
            f"{T} tokens scaled x{T / Ts:g}; {how}")
    return est, desc


def parity_summary(step, outputs):
    """The timed step's codes and sampled outputs against the oracle's (the
    oracle with its own statistics and scales, on the tokens of its sample).
    Every replica holds the same inputs, so the buffers of the last replay
    are the step's result."""
    import numpy as np
    import oracle
    wl = step.wl
    moved = total = 0
    worst = 0.0
    tokens = 0
    for g, _, Ls in step.groups:
        codes = step.codes[g].cpu().numpy().view(np.uint32)
        Y = step.Y[g].float().cpu().numpy()
        row = 0
        for L in Ls:
            oc, _, _, oy = outputs[L.name]
            gq = oracle.unpack_codes(codes[row:row + L.N, :oc.shape[1]], L.K,
                                     wl.bits)
            moved += int(np.count_nonzero(gq != oracle.unpack_codes(
                oc, L.K, wl.bits)))
            total += gq.size
            tokens = oy.shape[0]
            ys = Y[:tokens, row:row + L.N].astype(np.float64)
            worst = max(worst, float(np.linalg.norm(ys - oy) /
                                     max(np.linalg.norm(oy), 1e-300)))
            row += L.N
    return {"codes_differing": moved, "codes": total,
            "y_tokens": tokens, "y_rel_fro_max": worst}


# -------------------------------------------------------- aggregation ----

def slowest_rank_ms(ms: float, world: int, device) -> float:
    """The timed region's length on the slowest rank (all-reduce MAX)."""
    if world <= 1:
        return ms
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def layer_tokens_per_s(world: int, n_layers: int, T: int,
                       ms_per_step: float) -> float:
    """Whole-job prompt tokens per second per layer: every rank runs its own
    replica, so the job moves world * n_layers * T layer-tokens per step."""
    return world * n_layers * T / (ms_per_step / 1e3)


# ---------------------------------------------------------------- main ----

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def run_reference(args, wl):
    """The oracle as it stands, on the host cores, each step a bounded
    sample of the workload. A step takes a fraction of a second here, so the
    run stops after REFERENCE_SECONDS (at least three steps) even when more
    steps were asked for; the line gives the steps it timed."""
    torch.set_num_threads(1)
    data = make_inputs(wl)
    sample = 16
    cores = host_cores()
    for _ in range(min(args.warmup, 3)):
        oracle_step(wl, data, sample, cores)
    times = []
    desc = ""
    t0 = time.perf_counter()
    while len(times) < args.steps and (
            len(times) < 3 or time.perf_counter() - t0 < REFERENCE_SECONDS):
        est, desc = oracle_step(wl, data, sample, cores)
        times.append(est)
    wall = time.perf_counter() - t0
    per_step = sum(times) / len(times)
    value = len(wl.layers) * wl.T / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": len(times),
        "steps_requested": args.steps, "warmup": min(args.warmup, 3),
        "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "T": wl.T, "bits": wl.bits,
                   "group": wl.group, "layers": len(wl.layers)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


# The sources a kernel's counters depend on (its file and the headers it
# includes from the package).
KERNEL_SOURCES = {
    "gemm": ("gemm.cu", "common.cuh", "kperm.cuh"),
    "stats_scales": ("stats.cu", "awq_scale.cuh", "common.cuh"),
    "quantize": ("quantize.cu", "common.cuh"),
    "prepare": ("gemm.cu", "common.cuh", "kperm.cuh"),
}


def _code_only(text):
    """Source text without comments and whitespace (what compiles)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return re.sub(r"\s+", "", text)


def kernel_source_hash(kind="gemm"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "test_weight_quantization_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:12]


def traffic_from_profiles(kind, workload):
    """DRAM bytes per launch (read + write, averaged over one step's
    launches) of a kernel from a committed ncu summary, or None when absent
    or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kind}/{workload}")
    if (not e or kind not in KERNEL_SOURCES or
            e.get("source_hash") != kernel_source_hash(kind)):
        return None
    return e["dram_bytes_per_step"] / max(1, e.get("launches_per_step", 1))


def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return
    from test_weight_quantization_b200 import ttq
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    data = make_inputs(wl)

    probe = Step(ttq, wl, data, device, 1, args.separate)
    rep = max(2, math.ceil(2.5 * L2_BYTES / probe.input_bytes()))
    del probe
    step = Step(ttq, wl, data, device, rep, args.separate)
    stream = torch.cuda.Stream(device)
    torch.cuda.synchronize()

    # eager warm-up (loads kernels, sets attributes), then capture
    with torch.cuda.stream(stream):
        for r in range(rep):
            step.run(r)
    stream.synchronize()
    ttq.device_error(clear=True)
    kinds = [k for k, _ in step.plan]
    # external events record timestamps when replayed inside a graph
    ev = [[[torch.cuda.Event(enable_timing=True, external=not args.eager)
            for _ in range(2)] for _ in kinds] for _ in range(rep)]

    class Eager:
        def __init__(self, r, events=None):
            self.r, self.events = r, events

        def replay(self):
            step.run(self.r, self.events)

    graphs, igraphs = [], []
    for r in range(rep):
        if args.eager:
            graphs.append(Eager(r))
            igraphs.append(Eager(r, ev[r]))
            continue
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step.run(r)
        graphs.append(g)
        gi = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gi, stream=stream):
            step.run(r, ev[r])
        igraphs.append(gi)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            graphs[i % rep].replay()
    stream.synchronize()

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        clk.mark_start()
        with torch.cuda.stream(stream):
            start.record()
            for i in range(args.steps):
                graphs[i % rep].replay()
            end.record()
        torch.cuda.synchronize()
        clk.mark_end()
    barrier()
    ms = slowest_rank_ms(start.elapsed_time(end), world, device)
    clocks = clk.summary()
    ms_per_step = ms / args.steps
    value = layer_tokens_per_s(world, len(wl.layers), wl.T, ms_per_step)

    # per-kernel times: event-instrumented replays of the same step
    with torch.cuda.stream(stream):
        for r in range(rep):
            igraphs[r].replay()
    torch.cuda.synchronize()
    per_kind = {}
    for r in range(rep):
        for i, kind in enumerate(kinds):
            per_kind.setdefault(kind, 0.0)
            per_kind[kind] += ev[r][i][0].elapsed_time(ev[r][i][1]) / rep
    derr = ttq.device_error(clear=True)
    if derr:
        raise SystemExit(f"device error bits {derr:#x} raised during bench")

    pk = peaks()
    work = algorithmic_work(wl)
    kernels = {}
    for kind, msk in per_kind.items():
        e = {"ms_per_step": msk, "launches_per_step": kinds.count(kind)}
        if kind == "gemm":
            e["tflops"] = work["gemm_flops"] / (msk / 1e3) / 1e12
        e["gbs"] = work[kind] / (msk / 1e3) / 1e9
        kernels[kind] = e
    dom = max(per_kind, key=per_kind.get)
    if dom == "gemm":
        peak = pk["bf16_tflops_sustained"]
        achieved = kernels["gemm"]["tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": f"{pk['source']} bf16 sustained (fp16 dense rate "
                             "= bf16 nominal)"}
    else:
        peak = pk["hbm_gbs"]
        achieved = kernels[dom]["gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak,
                "peak_kind": f"{pk['source']} HBM copy"}
    roof["kernel"] = dom
    roof["traffic"] = traffic_from_profiles(dom, wl.name)
    roof["traffic_unit"] = "DRAM bytes per launch (ncu, cold serialised)"
    # algorithmic work of one launch, averaged over the step's launches
    n_dom = kinds.count(dom)
    roof["algorithmic_per_launch"] = (
        work["gemm_flops"] if dom == "gemm" else work[dom]) / max(1, n_dom)

    # end to end through the binding: host buffers in, host buffers out
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(ttq, wl, data, device, args, stream, world)

    cpu = cpu_one = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the unchanged oracle on every host core, and on one core
        cores = host_cores()
        outputs = {}
        est, desc = oracle_step(wl, data, ORACLE_SAMPLE_TOKENS, cores,
                                outputs)
        cpu = {"value": len(wl.layers) * wl.T / est, "unit": "tokens/s",
               "cores": cores, "kind": "oracle", "sample": desc}
        try:
            parity = parity_summary(step, outputs)
        except Exception as e:  # a report: never a reason to lose the line
            parity = {"error": repr(e)[:200]}
        if cores > 1:
            est, desc = oracle_step(wl, data, ORACLE_SAMPLE_TOKENS)
            cpu_one = {"value": len(wl.layers) * wl.T / est,
                       "unit": "tokens/s", "cores": 1, "kind": "oracle",
                       "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {
                "workload": wl.name, "T": wl.T, "bits": wl.bits,
                "group": wl.group,
                "layers": ", ".join(f"{L.name} {L.N}x{L.K}"
                                    for L in wl.layers),
                "projections": ", ".join(
                    f"{g} {step.N[g]}x{Ls[0].K}" for g, _, Ls in step.groups),
                "operands": "fp16 x fp16 -> fp32 (tensor cores); quantizer "
                            "fp32; statistics fp32",
                "l2": f"inputs rotate over {rep} replicas "
                      f"({rep * step.input_bytes() / 2**20:.0f} MiB > L2)",
                "parallelism": f"replicas x{world}",
                "launch": ("eager" if args.eager else
                           "CUDA graph per replica") + (
                    "; one stream, one call per step and layer"
                    if args.separate else
                    "; statistics+scales fused; prepare on a second stream "
                    "beside the quantizer")},
            "roofline": roof, "kernels": kernels,
            "gpu_launches": step.kernel_launches() * args.steps,
            "cpu_baseline": cpu, "cpu_baseline_one_core": cpu_one,
            "parity": parity, "e2e": e2e, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs, igraphs
        dist.destroy_process_group()


def end_to_end(ttq, wl, data, device, args, stream, world):
    """Same metric through the Python binding with host buffers: each step
    copies its prompt activations from pinned host memory, runs the path
    (eager calls, one per step of the method) and copies every output back.
    The layer weights are the model's resident parameters and stay on the
    device."""
    step = Step(ttq, wl, data, device, 1, args.separate)
    hx = {k: v.pin_memory() for k, v in data["X"].items()}
    hy = {g: torch.empty((wl.T, step.N[g]), dtype=wl.dtype).pin_memory()
          for g, _, _ in step.groups}
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = sum(v.numel() * v.element_size() for v in hy.values())

    def one():
        for k, v in hx.items():
            step.X[0][k].copy_(v, non_blocking=True)
        step.run(0)
        for n, v in hy.items():
            v.copy_(step.Y[n], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            one()
    stream.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    steps = max(5, args.steps // 2)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        a.record()
        for _ in range(steps):
            one()
        b.record()
    torch.cuda.synchronize()
    ms = slowest_rank_ms(a.elapsed_time(b) / steps, world, device)
    return {"value": layer_tokens_per_s(world, len(wl.layers), wl.T, ms),
            "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


if __name__ == "__main__":
    main()
