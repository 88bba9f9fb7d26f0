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
    """The reference arm times exactly the steps and warm-up asked for,
    reports the measured time per step, and prints the GPU arm's config."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--steps", "2", "--warmup",
                        "1", "--workload", "single-768"], capture_output=True,
                       text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1
    import bench
    from test_weight_quantization_b200.inputs import WORKLOADS
    assert line["config"] == bench.workload_config(WORKLOADS["single-768"], 1)
    # value is the sample's tokens over the measured time per step
    assert line["value"] == pytest.approx(
        1 * line["sample_tokens"] / (line["ms_per_step"] * 1e-3), rel=1e-9)
    assert line["ms_per_step"] * line["steps"] <= line["wall_s"] * 1e3 * (
        1 + 1e-9)
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == bench.host_cores()
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_roofline_peak_follows_the_timed_region():
    """A timed region under a second is compared with the burst tensor peak,
    a longer one with the sustained peak; frac is achieved / peak."""
    import bench
    pk = {"hbm_gbs": 6545.0, "bf16_tflops": 1627.8,
          "bf16_tflops_sustained": 1395.0, "source": "measured"}
    k = {"gemm": {"tflops": 1000.0, "gbs": 10.0}, "quantize": {"gbs": 5000}}
    short = bench.roofline("gemm", k, pk, 0.02)
    assert short["peak"] == 1627.8 and "burst" in short["peak_kind"]
    assert short["frac"] == pytest.approx(1000.0 / 1627.8)
    long = bench.roofline("gemm", k, pk, 3.0)
    assert long["peak"] == 1395.0 and "sustained" in long["peak_kind"]
    mem = bench.roofline("quantize", k, pk, 3.0)
    assert mem["bound"] == "hbm" and mem["frac"] == pytest.approx(5000 / 6545)


def test_default_workload_is_the_largest_single_gpu_configuration():
    import bench
    sys_argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        args = bench.parse()
    finally:
        sys.argv = sys_argv
    assert args.workload == "llama7b-prefill"
    from test_weight_quantization_b200.inputs import WORKLOADS
    wl = WORKLOADS[args.workload]
    # 3 layers of 4096 tokens; inputs of 154 MiB and weights of 212 MiB per
    # replica, two replicas > 2.5 x L2
    assert bench.input_bytes(wl) == 2 * 4096 * (4096 + 4096 + 11008) + \
        2 * (4096 * 4096 + 2 * 11008 * 4096)
    assert bench.replicas_for(wl) * bench.input_bytes(wl) >= \
        2.5 * bench.L2_BYTES


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
    """The bench line's parity report on a stand-in step whose buffers hold
    the oracle's own results: zero differences; one changed code and one
    changed output are seen."""
    import dataclasses
    import numpy as np
    import torch
    import bench
    import oracle
    from test_weight_quantization_b200 import ttq
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    base = WORKLOADS["opt125m-block"]
    wl = dataclasses.replace(base, T=64, layers=base.layers[:4])
    data = make_inputs(wl)

    class FakeStep:
        pass
    st = FakeStep()
    st.wl, st.groups = wl, bench.projection_groups(wl)
    st.inputs = bench.layer_inputs(wl)
    st.X = [dict(data["X"])]
    st.sums, st.s, st.inv = {}, {}, {}
    for k in st.inputs:
        X = data["X"][k].float().numpy()
        sums = oracle.act_sums(X).astype(np.float32)
        s, inv = oracle.awq_scales(sums.astype(np.float64), wl.T, wl.alpha,
                                   wl.lam, wl.p)
        st.sums[k] = torch.from_numpy(sums)
        st.s[k] = torch.from_numpy(s.astype(np.float32))
        st.inv[k] = torch.from_numpy(inv.astype(np.float32))
    st.W, st.N, st.codes, st.delta, st.zero, st.Y = [{}], {}, {}, {}, {}, {}
    for g, k, Ls in st.groups:
        K = Ls[0].K
        W = torch.cat([data["W"][L.name] for L in Ls])
        st.W[0][g], st.N[g] = W, W.shape[0]
        c, d, z = oracle.quantize(W.float().numpy(), st.s[k].numpy(),
                                  wl.bits, wl.group)
        cp = np.zeros((c.shape[0], ttq.codes_ld(K, wl.bits)), np.uint32)
        cp[:, :c.shape[1]] = c
        gl = ttq.groups_ld(K, wl.group)
        dp = np.zeros((c.shape[0], gl), np.float32)
        zp = np.zeros((c.shape[0], gl), np.uint8)
        dp[:, :d.shape[1]], zp[:, :z.shape[1]] = d, z
        st.codes[g] = torch.from_numpy(cp.view(np.int32))
        st.delta[g], st.zero[g] = torch.from_numpy(dp), torch.from_numpy(zp)
        y = oracle.lowbit_gemm(data["X"][k].float().numpy(),
                               st.inv[k].numpy(), c, d, z, W.shape[0],
                               wl.bits, wl.group)
        st.Y[g] = torch.from_numpy(y.astype(np.float32))
    assert [g for g, _, _ in st.groups] == ["q|k|v", "o"]
    rep = bench.parity_summary(st, threads=3, qrows=2304, ytokens=64)
    assert rep["codes_differing"] == 0 and rep["delta_differing"] == 0
    assert rep["codes"] == sum(L.N * L.K for L in wl.layers)
    assert rep["stats_rel_max"] < 1e-6 and rep["scales_rel_max"] < 1e-6
    assert rep["y_tokens"] == 64 and rep["y_rel_fro_max"] < 1e-6
    st.codes["q|k|v"][800, 0] ^= 1          # code 0 of row 32 of k
    st.Y["o"][3, 5] += 1.0
    rep = bench.parity_summary(st, threads=3, qrows=2304, ytokens=64)
    assert rep["codes_differing"] == 1
    assert rep["codes_differing_off_near_ties"] == 1
    assert rep["y_rel_fro_max"] > 1e-3


def test_clock_summary_keeps_the_samples_of_the_timed_region():
    """NVML samples (time, SM MHz, reason bits): the summary keeps the
    samples taken between the marks and names the active reasons; with none
    inside it falls back to all samples, flagged."""
    import bench
    samples = [(0.0, 1200.0, 0), (0.1, 1965.0, 0), (0.2, 1965.0, 0x4),
               (0.3, 1950.0, 0), (0.4, 1000.0, 0x8 | 0x40)]
    s = bench.ClockSampler.summarize(samples, 1965.0, 0.09, 0.31)
    assert s["samples"] == 3 and s["in_timed_region"]
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    s = bench.ClockSampler.summarize(samples, 1965.0, 9.0, 9.0)
    assert s["samples"] == 5 and not s["in_timed_region"]
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown",
                            "sw_power_cap"]
    assert bench.ClockSampler.summarize([], 1965.0) is None
