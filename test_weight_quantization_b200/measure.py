"""Per-kernel timing of the TTQ path on one GPU.

    python -m test_weight_quantization_b200.measure stats    T K [T K ...]
    python -m test_weight_quantization_b200.measure prepare  T K bits
    python -m test_weight_quantization_b200.measure quantize N K bits group
    python -m test_weight_quantization_b200.measure gemm     T N K bits group
    python -m test_weight_quantization_b200.measure qgemm    T N K bits group
    python -m test_weight_quantization_b200.measure lowrank  N K r iters
    python -m test_weight_quantization_b200.measure table    (the shapes below)
    python -m test_weight_quantization_b200.measure [--eager] KIND ...
        (--eager launches directly instead of replaying a CUDA graph)
    python -m test_weight_quantization_b200.measure decode   [T ...]
        (the decode sweep: 14336x4096 and 4096x14336, b in 2..5, g in
        16..128, at each T given; default T = 1 2 4 16)

Each call is captured REPS times in a CUDA graph and timed with CUDA events
around a replay, after three warm-up calls. Inputs are seeded and
synthetic (N(0, 1) activations, N(0, 0.02^2) weights, bf16). For the
memory-bound kernels (statistics, prepare, quantize, decode projection)
consecutive calls read different copies of the input, enough of them to
span 2.5x the L2 cache, so every call reads HBM. Rates are algorithmic
(every input read once, every output written once) and the fraction is
taken against MEASURED_PEAKS.json (HBM copy GB/s, or sustained bf16
TFLOP/s for the prefill projection). Prints one line per measurement.
"""
from __future__ import annotations

import json
import os
import sys

import torch

from test_weight_quantization_b200 import ttq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REPS = 20
L2_BYTES = 126 * 1024 * 1024


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d.get("bf16_tflops_sustained", d["bf16_tflops"])
    return 6650.0, 1400.0


EAGER = False  # --eager: launch directly instead of replaying a graph


def eager_us(fns):
    """Mean device time of one call, launched directly (for profilers)."""
    st = torch.cuda.Stream()
    n = max(REPS, len(fns))
    with torch.cuda.stream(st):
        for f in fns[:3]:
            f()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n):
            fns[i % len(fns)]()
        b.record()
    st.synchronize()
    return a.elapsed_time(b) / n * 1e3


def graph_us(fns):
    """Mean device time of one call, the calls in ``fns`` replayed in turn."""
    if EAGER:
        return eager_us(fns)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for f in fns[:3]:
            f()
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    n = max(REPS, len(fns))
    with torch.cuda.graph(g, stream=st):
        for i in range(n):
            fns[i % len(fns)]()
    with torch.cuda.stream(st):
        g.replay()
    st.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(st):
        a.record()
        g.replay()
        b.record()
    st.synchronize()
    return a.elapsed_time(b) / n * 1e3


def rotation(nbytes):
    """Copies of an operand of ``nbytes`` that together span 2.5x L2."""
    return max(1, min(64, -(-int(2.5 * L2_BYTES) // max(1, int(nbytes)))))


def _gen(seed):
    return torch.Generator(device="cuda").manual_seed(seed)


def acts(T, K, seed=1):
    return torch.randn(T, K, device="cuda", generator=_gen(seed)).to(
        torch.bfloat16)


def weights(N, K, seed=2):
    return (torch.randn(N, K, device="cuda", generator=_gen(seed)) * 0.02).to(
        torch.bfloat16)


def report(name, us, byts=None, flops=None):
    hbm, tf = peaks()
    if flops is not None:
        r = flops / us / 1e6
        print(f"{name}: {us:8.2f} us {r:8.1f} TF/s {r / tf:5.2f} of "
              f"{tf:.0f} TF/s", flush=True)
    else:
        r = byts / us / 1e3
        print(f"{name}: {us:8.2f} us {r:8.0f} GB/s {r / hbm:5.2f} of "
              f"{hbm:.0f} GB/s", flush=True)


def stats(T, K):
    Xr = [acts(T, K)]
    Xr += [Xr[0].clone() for _ in range(rotation(T * K * 2) - 1)]
    ctr = ttq.new_counter()
    sums = torch.empty(K, device="cuda")
    s = torch.empty_like(sums)
    inv = torch.empty_like(sums)
    us = graph_us([lambda X=X: ttq.act_stats(X, 2.0, out=sums) for X in Xr])
    report(f"stats          T={T:5d} K={K:6d}", us, T * K * 2 + K * 4)
    us = graph_us([lambda X=X: ttq.act_stats_scales(X, ctr, 0.5, 0.1, 2.0,
                                                    sums, s, inv)
                   for X in Xr])
    report(f"stats+scales   T={T:5d} K={K:6d}", us, T * K * 2 + K * 12)

    def two(X):
        ttq.act_stats(X, 2.0, out=sums)
        ttq.awq_scales(sums, T, 0.5, 0.1, 2.0, s, inv)
    us = graph_us([lambda X=X: two(X) for X in Xr])
    report(f"stats, scales  T={T:5d} K={K:6d} (two launches)", us,
           T * K * 2 + K * 12)


def prepare(T, K, bits):
    Xr = [acts(T, K)]
    Xr += [Xr[0].clone() for _ in range(rotation(T * K * 4) - 1)]
    inv = torch.ones(K, device="cuda")
    Xs = torch.empty(T, K, dtype=torch.float16, device="cuda")
    us = graph_us([lambda X=X: ttq.prepare_activations(X, inv, bits, None, Xs)
                   for X in Xr])
    report(f"prepare        T={T:5d} K={K:6d} b={bits}", us, T * K * 4 + K * 4)


def quantize(N, K, bits, group):
    Wr = [weights(N, K)]
    byts = N * K * 2 + K * 4 + N * K * bits // 8 + 5 * N * K // group
    Wr += [Wr[0].clone() for _ in range(rotation(byts) - 1)]
    s = torch.ones(K, device="cuda")
    c, d, z = ttq.quantize_rtn_grouped(Wr[0], s, bits, group)
    us = graph_us([lambda W=W: ttq.quantize_rtn_grouped(W, s, bits, group, c,
                                                        d, z) for W in Wr])
    report(f"quantize       N={N:6d} K={K:6d} b={bits} g={group:3d}", us, byts)


def gemm(T, N, K, bits, group):
    W = weights(N, K)
    X = acts(T, K)
    s = torch.ones(K, device="cuda")
    c, d, z = ttq.quantize_rtn_grouped(W, s, bits, group)
    del W
    Xs, _ = ttq.prepare_activations(X, s, bits)
    Y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    wbytes = N * K * bits / 8 + 5 * N * K / group
    copies = [(c, d, z)]
    if T <= 16:
        # decode: rotate the packed weights so that every call reads HBM
        n = max(2, rotation(wbytes))
        copies += [(c.clone(), d.clone(), z.clone()) for _ in range(n - 1)]
    fns = [lambda cc=cc, dd=dd, zz=zz: ttq.w_lowbit_gemm_prepared(
        Xs, None, cc, dd, zz, N, bits, group, out=Y) for cc, dd, zz in copies]
    us = graph_us(fns)
    name = f"gemm   T={T:5d} N={N:6d} K={K:6d} b={bits} g={group:3d}"
    if T <= 16:
        report(name, us, wbytes + 2 * T * (K + N))
    else:
        report(name, us, flops=2 * T * N * K)


TABLE = [
    ("stats", (4096, 4096)), ("stats", (4096, 11008)), ("stats", (2048, 768)),
    ("stats", (2048, 3072)),
    ("prepare", (4096, 4096, 4)), ("prepare", (4096, 11008, 4)),
    ("prepare", (2048, 768, 3)),
    ("quantize", (11008, 4096, 4, 128)), ("quantize", (4096, 4096, 4, 128)),
    ("quantize", (14336, 4096, 2, 16)), ("quantize", (2304, 768, 3, 32)),
    ("gemm", (4096, 11008, 4096, 4, 128)), ("gemm", (4096, 4096, 4096, 4, 128)),
    ("gemm", (1024, 6912, 1152, 4, 64)), ("gemm", (2048, 2304, 768, 3, 32)),
    ("gemm", (2048, 768, 3072, 3, 32)),
    ("gemm", (1, 14336, 4096, 4, 128)), ("gemm", (1, 4096, 14336, 5, 16)),
    ("gemm", (4, 14336, 4096, 4, 128)), ("gemm", (16, 14336, 4096, 4, 128)),
    ("gemm", (16, 4096, 14336, 2, 16)),
]



def qgemm(T, N, K, bits, group):
    """Quantize + projection as two launches against the fused launch that
    quantizes the bf16 weights inside the projection (codes stored)."""
    W = weights(N, K)
    X = acts(T, K)
    s = torch.ones(K, device="cuda")
    Xs, _ = ttq.prepare_activations(X, s, bits)
    c, d, z = ttq.quantize_rtn_grouped(W, s, bits, group)
    Y = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")

    def two():
        ttq.quantize_rtn_grouped(W, s, bits, group, c, d, z)
        ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, N, bits, group, out=Y)

    def fused():
        ttq.quantize_gemm_prepared(W, s, Xs, None, bits, group, out=Y,
                                   codes=c, delta=d, zero=z)
    flops = 2 * T * N * K
    name = f"T={T:5d} N={N:6d} K={K:6d} b={bits} g={group:3d}"
    report("quantize+gemm  " + name, graph_us([two]), flops=flops)
    report("fused qdq gemm " + name, graph_us([fused]), flops=flops)


def lowrank(N, K, r, iters):
    """Per-prompt low-rank factors (randomized subspace iteration, iters
    rounds) and the residual W - B A of an N x K bf16 weight. Algorithmic
    bytes of the factors: 2 + 2 iters reads of W; of the residual: W read
    and R written."""
    Wr = [weights(N, K)]
    Wr += [Wr[0].clone() for _ in range(rotation(N * K * 2) - 1)]
    s = torch.ones(K, device="cuda")
    om = torch.randn(r, K, device="cuda", generator=_gen(3))
    ws = torch.empty(ttq.lowrank_factors_workspace_size(N, K, r),
                     dtype=torch.uint8, device="cuda")
    B, A = ttq.lowrank_factors(Wr[0], s, om, iters, workspace=ws)
    R = torch.empty_like(Wr[0])
    name = f"N={N:6d} K={K:6d} r={r:2d}"
    us = graph_us([lambda W=W: ttq.lowrank_factors(W, s, om, iters,
                                                   workspace=ws)
                   for W in Wr])
    report(f"lowrank factors {name} iters={iters}", us,
           (2 + 2 * iters) * N * K * 2 + (N + K) * r * 2)
    us = graph_us([lambda W=W: ttq.lowrank_residual(W, B, A, out=R)
                   for W in Wr])
    report(f"lowrank residual {name}", us, 4 * N * K + (N + K) * r * 2)


def decode(*Ts):
    """The decode sweep's shapes at the given token counts."""
    for T in Ts or (1, 2, 4, 16):
        for N, K in ((14336, 4096), (4096, 14336)):
            for bits in (2, 3, 4, 5):
                for group in (16, 32, 64, 128):
                    gemm(T, N, K, bits, group)
                    torch.cuda.empty_cache()


FNS = {"stats": stats, "prepare": prepare, "quantize": quantize, "gemm": gemm,
       "qgemm": qgemm, "lowrank": lowrank}


def main(argv):
    global EAGER
    if argv and argv[0] == "--eager":
        EAGER = True
        argv = argv[1:]
    if argv and argv[0] == "decode":
        decode(*[int(a) for a in argv[1:]])
        return
    if not argv or argv[0] == "table":
        for kind, args in TABLE:
            FNS[kind](*args)
            torch.cuda.empty_cache()
        return
    kind, nums = argv[0], [int(a) for a in argv[1:]]
    fn = FNS[kind]
    arity = fn.__code__.co_argcount
    for i in range(0, len(nums), arity):
        fn(*nums[i:i + arity])


if __name__ == "__main__":
    main(sys.argv[1:])
