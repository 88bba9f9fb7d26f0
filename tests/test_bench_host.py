"""Host logic of bench.py that needs no GPU: the multi-rank aggregation
(world size 2 over gloo on the CPU) and the reference arm's behaviour under
a launcher (rank 0 reports, other ranks exit without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    import torch
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.slowest_rank_ms(local_ms[rank], world, torch.device("cpu"))
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_slowest_rank_timing_over_gloo():
    world, port = 2, _free_port()
    local_ms = [3.0, 5.5]
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, local_ms, out), nprocs=world,
             join=True)
    assert out[0] == out[1] == 5.5


def test_layer_token_throughput_counts_every_replica():
    import bench
    # 2 ranks x 6 layers x 2048 tokens per 0.25 ms step
    assert bench.layer_tokens_per_s(2, 6, 2048, 0.25) == pytest.approx(
        2 * 6 * 2048 / 0.25e-3)
    assert bench.layer_tokens_per_s(1, 6, 2048, 0.5) == pytest.approx(
        6 * 2048 / 0.5e-3)


def test_projection_groups_stack_layers_that_share_an_input():
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS
    wl = WORKLOADS["opt125m-block"]
    g = bench.projection_groups(wl)
    assert [(n, k, sum(L.N for L in Ls)) for n, k, Ls in g] == [
        ("q|k|v", "attn_in", 2304), ("o", "attn_out", 768),
        ("fc1", "mlp_in", 3072), ("fc2", "mlp_mid", 768)]
    # every layer appears exactly once
    assert sorted(L.name for _, _, Ls in g for L in Ls) == sorted(
        L.name for L in wl.layers)
    assert len(bench.projection_groups(wl, separate=True)) == 6
    # low-rank layers keep their own factors: never stacked
    gem = WORKLOADS["gemma1b-mlp"]
    assert all(len(Ls) == 1 for _, _, Ls in bench.projection_groups(gem))


def test_launch_plan_follows_the_method_per_input():
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS
    wl = WORKLOADS["opt125m-block"]
    inputs = bench.layer_inputs(wl)
    assert inputs == ["attn_in", "attn_out", "mlp_in", "mlp_mid"]
    plan = bench.launch_plan(inputs, bench.projection_groups(wl))
    assert len(plan) == 16
    assert plan[:4] == [("stats_scales", "attn_in"), ("prepare", "attn_in"),
                        ("quantize", "q|k|v"), ("gemm", "q|k|v")]
    sep = bench.launch_plan(inputs, bench.projection_groups(wl, True), True)
    assert len(sep) == 4 * 3 + 6 * 2
    # each projection comes after its input's scales and prepare
    for p in (plan, sep):
        for i, (kind, key) in enumerate(p):
            if kind == "gemm":
                k = next(kk for g, kk, _ in bench.projection_groups(
                    wl, p is sep) if g == key)
                assert ("prepare", k) in p[:i]


def test_reference_arm_rank_nonzero_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True,
                       env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_reports_the_oracle():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--steps", "1", "--warmup",
                        "0"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    import bench
    assert line["cpu_baseline"]["cores"] == bench.host_cores()
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "opt125m-block"


def test_measure_table_shapes_meet_the_call_constraints():
    """Every shape the measurement CLI times is a valid call of the ABI
    (K a multiple of 32 and of g, b in 2..8, g in {16, 32, 64, 128})."""
    from test_weight_quantization_b200 import measure
    for kind, args in measure.TABLE:
        assert kind in measure.FNS
        if kind == "quantize":
            N, K, b, g = args
        elif kind == "gemm":
            T, N, K, b, g = args
            assert T >= 1
        else:
            continue
        assert K % 32 == 0 and K % g == 0 and 2 <= b <= 8
        assert g in (16, 32, 64, 128)


def test_algorithmic_work_closed_forms():
    """The roofline numerator: flops 2 T N K per layer (plus the low-rank
    slab), bytes read and written once, each distinct input counted once."""
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS
    wl = WORKLOADS["opt125m-block"]
    w = bench.algorithmic_work(wl)
    T = 2048
    nk = 4 * 768 * 768 + 3072 * 768 + 768 * 3072
    assert w["gemm_flops"] == 2 * T * nk
    # q, k, v share one input: four distinct inputs of K = 768, 768, 768, 3072
    kin = 768 + 768 + 768 + 3072
    assert w["stats"] == T * kin * 2 + kin * 4
    assert w["prepare"] == T * kin * 4 + kin * 4
    assert w["stats_scales"] == w["stats"] + w["scales"]
    # quantize: bf16 W in, b/8 bytes of codes and 5/g bytes of params out
    assert w["quantize"] == sum(L.N * L.K * 2 + L.K * 4 + L.N * L.K * 3 // 8 +
                                5 * L.N * L.K // 32 for L in wl.layers)
    gem = WORKLOADS["gemma1b-mlp"]
    wg = bench.algorithmic_work(gem)
    assert wg["gemm_flops"] == sum(2 * 1024 * L.N * L.K + 2 * 1024 * 16 *
                                   (L.K + L.N) for L in gem.layers)


def test_threaded_oracle_baseline_computes_the_same_step():
    """The all-cores CPU baseline runs the unchanged oracle on disjoint
    slices; its codes, scales and projection equal the one-thread run (the
    partial channel sums only change the fp64 summation order)."""
    import dataclasses
    import numpy as np
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    for name in ("opt125m-block", "gemma1b-mlp"):
        base = WORKLOADS[name]
        wl = dataclasses.replace(base, T=96, layers=base.layers[:2])
        data = make_inputs(wl)
        one, many = {}, {}
        bench.oracle_step(wl, data, 8, threads=1, outputs=one)
        est, desc = bench.oracle_step(wl, data, 8, threads=5, outputs=many)
        assert est > 0 and "5 threads" in desc
        assert one.keys() == many.keys() == {L.name for L in wl.layers}
        for k in one:
            for a, b in zip(one[k][:3], many[k][:3]):
                assert np.array_equal(a, b)
            np.testing.assert_allclose(many[k][3], one[k][3], rtol=1e-12,
                                       atol=1e-12)
            assert one[k][3].shape == (8, next(L.N for L in wl.layers
                                                if L.name == k))


def test_host_cores_and_ranges_cover_the_work():
    import bench
    assert bench.host_cores() >= 1
    for n, parts in ((10, 3), (7, 7), (5, 9), (768, 224), (1, 1)):
        r = bench._ranges(n, parts)
        assert r[0][0] == 0 and r[-1][1] == n and len(r) == min(n, parts)
        assert all(a < b for a, b in r)
        assert all(r[i][1] == r[i + 1][0] for i in range(len(r) - 1))


def test_parity_summary_reads_the_step_buffers():
    """The bench line's parity report: the step's (stacked) codes and
    sampled outputs against the oracle's. Buffers equal to the oracle's give
    zero moved codes and zero error; one changed code and one changed
    output are seen."""
    import dataclasses
    import numpy as np
    import torch
    import bench
    from test_weight_quantization_b200 import ttq
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    base = WORKLOADS["opt125m-block"]
    wl = dataclasses.replace(base, T=64, layers=base.layers[:4])
    data = make_inputs(wl)
    outputs = {}
    bench.oracle_step(wl, data, 8, 1, outputs)

    class FakeStep:
        pass
    st = FakeStep()
    st.wl, st.groups = wl, bench.projection_groups(wl)
    st.codes, st.Y = {}, {}
    for g, _, Ls in st.groups:
        K = Ls[0].K
        c = np.concatenate([outputs[L.name][0] for L in Ls])
        padded = np.zeros((c.shape[0], ttq.codes_ld(K, wl.bits)), np.uint32)
        padded[:, :c.shape[1]] = c
        st.codes[g] = torch.from_numpy(padded.view(np.int32))
        y = np.concatenate([outputs[L.name][3] for L in Ls], axis=1)
        st.Y[g] = torch.from_numpy(y.astype(np.float32))
    assert [g for g, _, _ in st.groups] == ["q|k|v", "o"]
    rep = bench.parity_summary(st, outputs)
    assert rep["codes_differing"] == 0
    assert rep["codes"] == sum(L.N * L.K for L in wl.layers)
    assert rep["y_tokens"] == 8 and rep["y_rel_fro_max"] < 1e-6
    st.codes["q|k|v"][800, 0] ^= 1          # code 0 of row 32 of k
    st.Y["o"][3, 5] += 1.0
    rep = bench.parity_summary(st, outputs)
    assert rep["codes_differing"] == 1 and rep["y_rel_fro_max"] > 1e-3


def test_clock_summary_keeps_the_samples_of_the_timed_region():
    """nvidia-smi rows (timestamp first): the summary keeps the rows taken
    between the marks, and falls back to all rows, flagged, if none are."""
    import datetime
    import bench
    base = datetime.datetime(2026, 1, 2, 3, 4, 5)

    def row(ms, mhz, cap="Not Active"):
        ts = (base + datetime.timedelta(milliseconds=ms)).strftime(
            "%Y/%m/%d %H:%M:%S.%f")[:-3]
        return (f"{ts}, 0, {mhz}, 1965, 700.5, 0x0, Not Active, Not Active, "
                f"Not Active, {cap}\n")
    lines = [row(0, 1200), row(100, 1965), row(200, 1965, "Active"),
             row(300, 1950), row(400, 1000)]
    t0 = base + datetime.timedelta(milliseconds=90)
    t1 = base + datetime.timedelta(milliseconds=310)
    s = bench.ClockSampler.summarize(lines, t0, t1)
    assert s["samples"] == 3 and s["in_timed_region"]
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    late = base + datetime.timedelta(seconds=9)
    s = bench.ClockSampler.summarize(lines, late, late)
    assert s["samples"] == 5 and not s["in_timed_region"]
    assert bench.ClockSampler.summarize(["garbage\n"]) is None
