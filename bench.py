#!/usr/bin/env python3
"""Throughput of the TTQ hot path: prompt tokens/s per layer, including the
on-the-fly quantization.

One step is one pass of the whole path over one prompt of the workload: for
every distinct layer input, statistics and scales (one launch) -> prepared
fp16 operand; for every layer, group RTN of its weight -> tensor-core
low-bit projection. Layers that share an input run as one projection of
their stacked weights, and the prepared operand is built on a second stream
while the weights are quantized. The default workload is the largest one
that fits one GPU: Llama-7B-shaped prefill layers (attn 4096x4096, up
11008x4096, down 4096x11008), T = 4096, b = 4, g = 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

With N > 1 (launched by torchrun) every rank runs an independent replica
(the path has no exchange step), the timed region is bracketed by a barrier
and a device synchronisation, and the slowest rank's time counts.
Rank 0 prints one JSON line. ``--impl reference`` times the CPU oracle
instead (rank 0 only), each step the whole path on a bounded prompt sample.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs  # noqa

METRIC = "prompt tokens/s per layer incl. on-the-fly quant"
L2_BYTES = 126 * 1024 * 1024
# prompt tokens of the oracle's sample step (the whole path on a prompt of
# this many tokens of the workload's inputs)
ORACLE_SAMPLE_TOKENS = 128
# the oracle's CPU baseline repeats its sample step for at least this long
CPU_BASELINE_SECONDS = 10.0
# the reference arm shrinks its sample so that warm-up and steps together
# take about this long
REFERENCE_BUDGET_SECONDS = 150.0
# a timed region at least this long is compared with the sustained tensor
# peak, a shorter one with the burst peak
SUSTAINED_REGION_SECONDS = 1.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # about 1 ms per Llama-sized step: 1000 steps take about a second
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b-prefill",
                    choices=sorted(w for w in WORKLOADS
                                   if w != "decode-sweep"))
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
    """Samples the SM clock and the active clock-event (throttle) reasons of
    one GPU through NVML every ``period`` seconds on a background thread
    (read-only queries). The summary keeps the samples taken between
    mark_start() and mark_end(); if none fell inside, all samples, flagged.
    """
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, cuda_index, period=0.002):
        self.cuda_index = cuda_index
        self.period = period
        self.samples = []      # (monotonic seconds, sm MHz, reason bits)
        self.max_mhz = None
        self.t0 = self.t1 = None
        self._stop = None
        self._thread = None
        self._nvml = None

    def _handle(self, nvml):
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        import threading
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            h = self._handle(nvml)
            self.max_mhz = float(nvml.nvmlDeviceGetMaxClockInfo(
                h, nvml.NVML_CLOCK_SM))
        except Exception:
            return self
        self._nvml = nvml
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    mhz = nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM)
                    bits = nvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    break
                self.samples.append((time.monotonic(), float(mhz), int(bits)))
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()
        time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def summary(self):
        if self.max_mhz is None:
            return None
        return self.summarize(self.samples, self.max_mhz, self.t0, self.t1)

    @classmethod
    def summarize(cls, samples, max_mhz, t0=None, t1=None):
        """Median SM clock, the maximum clock and the active reasons of the
        samples (time, MHz, reason bits) that fall in [t0, t1]."""
        if not samples:
            return None
        inside = samples
        if t0 is not None and t1 is not None:
            inside = [x for x in samples if t0 <= x[0] <= t1]
        use = inside if inside else samples
        reasons = sorted({name for _, _, bits in use
                          for name, bit in cls.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(x[1] for x in use),
                "sm_max_mhz": max_mhz, "samples": len(use),
                "in_timed_region": bool(inside), "reasons": reasons,
                "source": "NVML, every %g ms" % (cls_period_ms(use))}


def cls_period_ms(samples):
    """Median spacing of the samples, in ms (0 for fewer than two)."""
    if len(samples) < 2:
        return 0.0
    gaps = [b[0] - a[0] for a, b in zip(samples, samples[1:])]
    return round(statistics.median(gaps) * 1e3, 2)


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


def oracle_step(wl, data, tokens, threads=1, outputs=None):
    """The CPU oracle on a bounded sample of one step: the whole path for a
    prompt made of the first ``tokens`` tokens of every layer input
    (statistics and scales over those tokens, group RTN of the full
    weights, projection of those tokens). Returns (seconds, description).

    With ``threads`` > 1 the unchanged oracle functions run concurrently on
    disjoint slices: the statistics over token ranges (the partial sums are
    added), the quantizer and the projection over output rows. The C calls
    release the GIL. ``outputs``, when a dict, receives every layer's
    (codes, delta, zero, Y) for checking."""
    import numpy as np
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    Ts = min(tokens, wl.T)
    Xn = {k: v[:Ts].float().numpy() for k, v in data["X"].items()}
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
            sums = sum(each(lambda a, b: oracle.act_sums(X[a:b], wl.p), Ts))
            s[k], inv[k] = oracle.awq_scales(sums, Ts, wl.alpha, wl.lam, wl.p)
        for L in wl.layers:
            W = data["W"][L.name].float().numpy()
            s32 = s[L.input_name].astype(np.float32)
            parts = each(lambda a, b: oracle.quantize(W[a:b], s32, wl.bits,
                                                      wl.group), L.N)
            c, d, z = (np.concatenate(x) for x in zip(*parts))
            A = B = None
            if wl.rank:
                A = data["A"][L.name].float().numpy()
                B = data["B"][L.name].float().numpy()
            X = Xn[L.input_name]
            ys = each(lambda a, b: oracle.lowbit_gemm(
                X, inv[L.input_name], c[a:b], d[a:b], z[a:b], b - a, wl.bits,
                wl.group, A, None if B is None else B[a:b]), L.N)
            if outputs is not None:
                outputs[L.name] = (c, d, z, np.concatenate(ys, axis=1))
        seconds = time.perf_counter() - t0
    finally:
        if pool is not None:
            pool.shutdown()
    how = ("1 thread" if threads == 1 else
           f"{threads} threads on disjoint token ranges (statistics) and "
           f"output rows (quantizer, projection)")
    desc = (f"the whole path (statistics, scales, group RTN of the full "
            f"weights, projection) on a prompt of the first {Ts} of the "
            f"{wl.T} tokens; {how}")
    return seconds, desc


def cpu_baseline(wl, data, threads, min_seconds=CPU_BASELINE_SECONDS,
                 tokens=ORACLE_SAMPLE_TOKENS):
    """The oracle's sample step repeated for at least ``min_seconds`` (and
    at least twice); tokens/s per layer over the steps it ran."""
    times, desc = [], ""
    while len(times) < 2 or sum(times) < min_seconds:
        sec, desc = oracle_step(wl, data, tokens, threads)
        times.append(sec)
    Ts = min(tokens, wl.T)
    return {"value": len(wl.layers) * Ts * len(times) / sum(times),
            "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{desc}; {len(times)} steps, "
                      f"{sum(times):.1f} s"}


def parity_summary(step, threads=1, qrows=64, ytokens=8, seed=5):
    """The timed step's results against the oracle, on the step's own
    inputs and upstream outputs: the statistics of every input in full;
    the scales from the GPU's sums; for every projection the codes of
    ``qrows`` sampled weight rows (quantized by the oracle with the GPU's
    scales; bit-exact apart from the near-ties the oracle marks) and every
    output channel of ``ytokens`` sampled tokens (the oracle's projection
    of the GPU's codes). Every replica holds the same inputs, so the buffers
    of the last replay are the step's result."""
    import numpy as np
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    wl = step.wl
    rng = np.random.default_rng(seed)
    rep = {"stats_rel_max": 0.0, "scales_rel_max": 0.0, "codes": 0,
           "codes_differing": 0, "codes_differing_off_near_ties": 0,
           "weight_near_ties": 0, "zero_point_near_tie_groups": 0,
           "delta_differing": 0, "y_tokens": 0, "y_rel_fro_max": 0.0}

    def rel(a, b):
        b = np.asarray(b, np.float64)
        return float(np.max(np.abs(np.asarray(a, np.float64) - b) /
                            np.maximum(np.abs(b), 1e-30)))

    pool = ThreadPoolExecutor(threads) if threads > 1 else None
    try:
        for k in step.inputs:
            X = step.X[0][k].float().cpu().numpy()
            sums = step.sums[k].cpu().numpy()
            rep["stats_rel_max"] = max(rep["stats_rel_max"], rel(
                sums, oracle.act_sums(X, wl.p)))
            rs, _ = oracle.awq_scales(sums.astype(np.float64), wl.T,
                                      wl.alpha, wl.lam, wl.p)
            rep["scales_rel_max"] = max(rep["scales_rel_max"], rel(
                step.s[k].cpu().numpy(), rs))
        for g, k, Ls in step.groups:
            K = Ls[0].K
            N = step.N[g]
            W = step.W[0][g].float().cpu().numpy()
            s32 = step.s[k].cpu().numpy()
            inv32 = step.inv[k].cpu().numpy()
            words, G = K * wl.bits // 32, K // wl.group
            codes = step.codes[g].cpu().numpy().view(np.uint32)[:, :words]
            delta = step.delta[g].cpu().numpy()[:, :G]
            zero = step.zero[g].cpu().numpy()[:, :G]
            rows = np.sort(rng.choice(N, size=min(qrows, N), replace=False))
            rc, rd, rz = oracle.quantize(W[rows], s32, wl.bits, wl.group)
            mask, wt, gt = oracle.near_tie_mask(W[rows], s32, wl.bits,
                                                wl.group)
            diff = oracle.unpack_codes(codes[rows], K, wl.bits) != \
                oracle.unpack_codes(rc, K, wl.bits)
            rep["codes"] += diff.size
            rep["codes_differing"] += int(diff.sum())
            rep["codes_differing_off_near_ties"] += int(
                (diff & (mask == 0)).sum())
            rep["weight_near_ties"] += wt
            rep["zero_point_near_tie_groups"] += gt
            rep["delta_differing"] += int((delta[rows] != rd).sum())
            inner = np.arange(1, wl.T - 1)
            tok = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(
                inner, size=min(max(0, ytokens - 2), inner.size),
                replace=False)])).astype(np.int64)
            X = step.X[0][k].float().cpu().numpy()[tok]
            A = B = None
            if wl.rank:
                A = step.A[g].float().cpu().numpy()
                B = step.B[g].float().cpu().numpy()

            def part(ab):
                a, b = ab
                return oracle.lowbit_gemm(
                    X, inv32, codes[a:b], delta[a:b], zero[a:b], b - a,
                    wl.bits, wl.group, A, None if B is None else B[a:b])
            pieces = _ranges(N, threads)
            ys = list(pool.map(part, pieces)) if pool else \
                [part(ab) for ab in pieces]
            ref = np.concatenate(ys, axis=1)
            Y = step.Y[g].float().cpu().numpy()[tok].astype(np.float64)
            rep["y_tokens"] = len(tok)
            rep["y_rel_fro_max"] = max(rep["y_rel_fro_max"], float(
                np.linalg.norm(Y - ref) / max(np.linalg.norm(ref), 1e-300)))
    finally:
        if pool is not None:
            pool.shutdown()
    return rep


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
    """The oracle as it stands, on every host core, each step the whole path
    on a bounded prompt sample (ORACLE_SAMPLE_TOKENS tokens, the sample of
    the GPU arm's cpu_baseline). When warm-up and steps together would take
    longer than REFERENCE_BUDGET_SECONDS the sample shrinks in proportion,
    judged from one untimed calibration step. ms_per_step is the measured
    wall time per timed step; value is the tokens those steps processed per
    second per layer."""
    torch.set_num_threads(1)
    data = make_inputs(wl)
    cores = host_cores()
    tokens = min(ORACLE_SAMPLE_TOKENS, wl.T)
    t_cal, _ = oracle_step(wl, data, tokens, cores)
    total = (args.steps + args.warmup) * t_cal
    if total > REFERENCE_BUDGET_SECONDS:
        tokens = max(1, int(tokens * REFERENCE_BUDGET_SECONDS / total))
    for _ in range(args.warmup):
        oracle_step(wl, data, tokens, cores)
    times, desc = [], ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sec, desc = oracle_step(wl, data, tokens, cores)
        times.append(sec)
    wall = time.perf_counter() - t0
    per_step = wall / max(1, len(times))
    value = len(wl.layers) * tokens / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": len(times),
        "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "sample_tokens": tokens, "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


def input_bytes(wl):
    """Bytes of one replica's inputs: every distinct layer input and every
    weight, at the workload's storage type."""
    xb = 4 if wl.dtype == torch.float32 else 2
    ks = {L.input_name: L.K for L in wl.layers}
    return (sum(wl.T * K * xb for K in ks.values()) +
            sum(L.N * L.K * xb for L in wl.layers) +
            sum(wl.rank * (L.N + L.K) * xb for L in wl.layers))


def replicas_for(wl):
    """Input replicas the timed loop rotates over: together at least 2.5x
    the L2 cache, so every step reads its inputs from HBM."""
    return max(2, math.ceil(2.5 * L2_BYTES / input_bytes(wl)))


def workload_config(wl, n_gpus):
    """The ``config`` of the JSON line (both arms print the same)."""
    rep = replicas_for(wl)
    return {
        "workload": wl.name, "T": wl.T, "bits": wl.bits, "group": wl.group,
        "alpha": wl.alpha, "lambda": wl.lam, "p": wl.p, "rank": wl.rank,
        "layers": ", ".join(f"{L.name} {L.N}x{L.K}" for L in wl.layers),
        "projections": ", ".join(f"{g} {sum(L.N for L in Ls)}x{Ls[0].K}"
                                 for g, _, Ls in projection_groups(wl)),
        "operands": "fp16 x fp16 -> fp32 (tensor cores); quantizer fp32; "
                    "statistics fp32",
        "l2": f"inputs rotate over {rep} replicas "
              f"({rep * input_bytes(wl) / 2**20:.0f} MiB > L2)",
        "parallelism": f"independent replicas x{n_gpus}",
    }


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

    rep = replicas_for(wl)
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
    region_s = ms / 1e3
    roof = roofline(dom, kernels, pk, region_s)
    roof["traffic"] = traffic_from_profiles(dom, wl.name)
    roof["traffic_unit"] = "DRAM bytes per launch (ncu, cold serialised)"
    # algorithmic work of one launch, averaged over the step's launches
    n_dom = kinds.count(dom)
    roof["algorithmic_per_launch"] = (
        work["gemm_flops"] if dom == "gemm" else work[dom]) / max(1, n_dom)
    roof["timed_region_s"] = region_s

    # end to end through the binding: host buffers in, host buffers out
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(ttq, wl, data, device, args, world)

    cpu = parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = host_cores()
        try:
            parity = parity_summary(step, cores)
        except Exception as e:  # a report: never a reason to lose the line
            parity = {"error": repr(e)[:200]}
        # the unchanged oracle on every host core
        cpu = cpu_baseline(wl, data, cores)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "config": workload_config(wl, world),
            "launch": ("eager" if args.eager else
                       "CUDA graph per replica") + (
                "; one stream, one call per step and layer"
                if args.separate else
                "; statistics+scales fused; prepare on a second stream "
                "beside the quantizer"),
            "roofline": roof, "kernels": kernels,
            "gpu_launches": step.kernel_launches() * args.steps,
            "cpu_baseline": cpu, "parity": parity, "e2e": e2e,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        del graphs, igraphs
        dist.destroy_process_group()


def roofline(dom, kernels, pk, region_s):
    """The roofline object of the dominant kernel. A tensor-core kernel is
    compared with the measured bf16 burst peak when the timed region is
    shorter than SUSTAINED_REGION_SECONDS and with the sustained peak
    otherwise (fp16 has the same dense rate as bf16)."""
    if dom == "gemm":
        sustained = region_s >= SUSTAINED_REGION_SECONDS
        peak = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
        achieved = kernels["gemm"]["tflops"]
        return {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "kernel": dom,
                "peak_kind": f"{pk['source']} bf16 "
                             f"{'sustained' if sustained else 'burst'} "
                             f"(timed region {region_s:.3g} s; fp16 dense "
                             f"rate = bf16)"}
    peak = pk["hbm_gbs"]
    achieved = kernels[dom]["gbs"]
    return {"bound": "hbm", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak, "kernel": dom,
            "peak_kind": f"{pk['source']} HBM copy"}


def end_to_end(ttq, wl, data, device, args, world):
    """Same metric through the Python binding with host buffers: each step
    copies its prompt activations from pinned host memory, runs the path
    (eager calls, one per step of the method) and copies every output back
    to pinned host memory. The layer weights are the model's resident
    parameters and stay on the device. Steps are pipelined over two buffer
    sets: the copy-in of step i+1 and the copy-out of step i-1 run on their
    own streams while step i computes. Every byte of every step still
    crosses PCIe inside the timed region."""
    sets = [Step(ttq, wl, data, device, 1, args.separate) for _ in range(2)]
    hx = {k: v.pin_memory() for k, v in data["X"].items()}
    hy = [{g: torch.empty((wl.T, sets[0].N[g]), dtype=wl.dtype).pin_memory()
           for g, _, _ in sets[0].groups} for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in hx.values())
    d2h = sum(v.numel() * v.element_size() for v in hy[0].values())
    comp = torch.cuda.Stream(device)
    cin = torch.cuda.Stream(device)
    cout = torch.cuda.Stream(device)
    free_in = [None, None]    # compute of the set's last step done
    free_out = [None, None]   # copy-out of the set's last step done

    def one(i):
        b = i % 2
        st = sets[b]
        with torch.cuda.stream(cin):
            if free_in[b] is not None:
                cin.wait_event(free_in[b])
            for k, v in hx.items():
                st.X[0][k].copy_(v, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(cin)
        with torch.cuda.stream(comp):
            comp.wait_event(loaded)
            if free_out[b] is not None:
                comp.wait_event(free_out[b])
            st.run(0)
            done = torch.cuda.Event()
            done.record(comp)
        free_in[b] = done
        with torch.cuda.stream(cout):
            cout.wait_event(done)
            for n, v in hy[b].items():
                v.copy_(st.Y[n], non_blocking=True)
            out = torch.cuda.Event()
            out.record(cout)
        free_out[b] = out

    for i in range(max(3, args.warmup)):
        one(i)
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 200))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(cin)
    for i in range(steps):
        one(i)
    # the region ends when the last copy-out has landed
    torch.cuda.current_stream().wait_stream(cout)
    torch.cuda.current_stream().wait_stream(comp)
    b.record(torch.cuda.current_stream())
    torch.cuda.synchronize()
    ms = slowest_rank_ms(a.elapsed_time(b) / steps, world, device)
    return {"value": layer_tokens_per_s(world, len(wl.layers), wl.T, ms),
            "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "copy-in, compute and copy-out on three streams "
                         "over two buffer sets"}


if __name__ == "__main__":
    main()
