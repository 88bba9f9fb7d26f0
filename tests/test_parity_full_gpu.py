"""GPU parity at the full sizes of every workload, in the launch
configuration the benchmark times (prepare + tensor-core projection, bf16 or
fp32 output as the workload stores it).

Statistics and scales are compared in full; quantization bit for bit on all
rows (small layers) or on sampled rows (large ones); the projection on
sampled token rows (first, last and seeded picks) with every output channel.
Sampling keeps the fp64 oracle to seconds per layer.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_codes_match, assert_gemm_close,
                         assert_rel_close, np32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ttq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_weight_quantization_b200 import ttq as mod
    mod.device_error(clear=True)
    yield mod
    assert mod.device_error(clear=True) == 0


def sample_rows(n, k, seed):
    rng = np.random.default_rng(seed)
    extra = rng.choice(np.arange(1, n - 1), size=max(0, k - 2), replace=False)
    return np.unique(np.concatenate([[0, n - 1], extra])).astype(np.int64)


def dense(c, d, z, K, bits, group, rows=None):
    c = c.cpu().numpy().view(np.uint32)
    d, z = d.cpu().numpy(), z.cpu().numpy()
    if rows is not None:
        c, d, z = c[rows], d[rows], z[rows]
    return (c[:, :K * bits // 32], d[:, :K // group], z[:, :K // group])


def check_layer(ttq, wl, name, X, W, A, B, bits, group, T_tok, qrows,
                ytok, seed):
    """One layer: GPU path on full tensors, oracle on samples."""
    Xg, Wg = X.cuda(), W.cuda()
    K = X.shape[1]
    N = W.shape[0]
    sums = ttq.act_stats(Xg, wl.p)
    assert_rel_close(np32(sums), oracle.act_sums(np32(X), wl.p),
                     what=f"{name} sums")
    s, inv = ttq.awq_scales(sums, X.shape[0], wl.alpha, wl.lam, wl.p)
    rs, rinv = oracle.awq_scales(np32(sums).astype(np.float64), X.shape[0],
                                 wl.alpha, wl.lam, wl.p)
    assert_rel_close(np32(s), rs, what=f"{name} s")
    assert_rel_close(np32(inv), rinv, what=f"{name} inv_s")
    c, d, z = ttq.quantize_rtn_grouped(Wg, s, bits, group)
    rows = None if qrows is None else sample_rows(N, qrows, seed)
    Wn = np32(W) if rows is None else np32(W)[rows]
    rc, rd, rz = oracle.quantize(Wn, np32(s), bits, group)
    gc, gd, gz = dense(c, d, z, K, bits, group, rows)
    assert_codes_match(gc, gd, gz, rc, rd, rz, Wn, np32(s), bits, group,
                       f"{name} codes")
    # the oracle's own scales (fp64, stored as fp32) differ from the GPU's by
    # an fp32 ulp or two on some channels; codes may move only where that
    # shifts w*s/D across a rounding boundary, a few per million
    oc, _, _ = oracle.quantize(Wn, rs.astype(np.float32), bits, group)
    moved = int(np.count_nonzero(oracle.unpack_codes(oc, K, bits) !=
                                 oracle.unpack_codes(rc, K, bits)))
    print(f"{name}: {moved} of {Wn.size} codes differ with the oracle's s")
    assert moved <= max(16, 1e-4 * Wn.size), f"{name}: {moved} codes moved"
    # projection of the first T_tok tokens, as the benchmark launches it
    Xt = Xg[:T_tok]
    Ag = None if A is None else A.cuda()
    Bg = None if B is None else B.cuda()
    Xs, U = ttq.prepare_activations(Xt, inv, bits, Ag)
    Y = ttq.w_lowbit_gemm_prepared(Xs, U, c, d, z, N, bits, group, Bg,
                                   out_dtype=wl.dtype)
    torch.cuda.synchronize()
    tok = sample_rows(T_tok, ytok, seed + 1) if T_tok > ytok else \
        np.arange(T_tok)
    cd, dd, zd = dense(c, d, z, K, bits, group)
    ref = oracle.lowbit_gemm(np32(X[:T_tok]), np32(inv), cd, dd, zd, N, bits,
                             group, None if A is None else np32(A),
                             None if B is None else np32(B), rows=tok)
    assert_gemm_close(np32(Y)[tok], ref, f"{name} projection", Y.dtype)
    return c, d, z, inv


@pytest.mark.parametrize("wname", ["single-768", "opt125m-block",
                                   "gemma1b-mlp", "llama7b-prefill"])
def test_workload_full_size(ttq, wname):
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS[wname]
    data = make_inputs(wl)
    big = wname == "llama7b-prefill"
    for li, layer in enumerate(wl.layers):
        X = data["X"][layer.input_name]
        W = data["W"][layer.name]
        A = data["A"].get(layer.name)
        B = data["B"].get(layer.name)
        check_layer(ttq, wl, f"{wname}/{layer.name}", X, W, A, B, wl.bits,
                    wl.group, wl.T, 48 if big else None, 6 if big else 16,
                    7 * li + 3)


def test_decode_sweep_full_size(ttq):
    """Weights quantized once from a 512-token prompt, then projections at
    T = 1, 4, 16 for every (b, g) of the decode sweep."""
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["decode-sweep"]
    data = make_inputs(wl)
    for bits in wl.extra["bits"]:
        for group in wl.extra["groups"]:
            for li, layer in enumerate(wl.layers):
                X = data["X"][layer.input_name]
                W = data["W"][layer.name]
                Xg = X.cuda()
                sums = ttq.act_stats(Xg)
                s, inv = ttq.awq_scales(sums, X.shape[0])
                c, d, z = ttq.quantize_rtn_grouped(W.cuda(), s, bits, group)
                rows = sample_rows(layer.N, 24, bits * 100 + group)
                Wn = np32(W)[rows]
                rc, rd, rz = oracle.quantize(Wn, np32(s), bits, group)
                gc, gd, gz = dense(c, d, z, layer.K, bits, group, rows)
                assert_codes_match(gc, gd, gz, rc, rd, rz, Wn, np32(s), bits,
                                   group, f"decode b={bits} g={group} "
                                   f"{layer.name}")
                cd, dd, zd = dense(c, d, z, layer.K, bits, group)
                # one decode width per (b, g, layer) keeps the oracle short;
                # across the sweep every width meets every layer
                T = (1, 4, 16)[(bits + group // 16 + li) % 3]
                Xs, _ = ttq.prepare_activations(Xg[:T], inv, bits)
                Y = ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, layer.N,
                                               bits, group)
                torch.cuda.synchronize()
                tok = np.arange(T) if T <= 2 else np.array([0, T - 1])
                ref = oracle.lowbit_gemm(np32(X[:T]), np32(inv), cd, dd, zd,
                                         layer.N, bits, group, rows=tok)
                assert_gemm_close(np32(Y)[tok], ref,
                                  f"decode b={bits} g={group} T={T} "
                                  f"{layer.name}", Y.dtype)


def test_stacked_projection_matches_layers(ttq):
    """q, k, v of the OPT block as one projection of their stacked weights
    (as the benchmark runs them): codes equal the per-layer codes row for
    row, outputs equal the per-layer outputs column block for column block,
    and the fused statistics + scales launch feeds both."""
    from test_weight_quantization_b200.inputs import WORKLOADS, make_inputs
    wl = WORKLOADS["opt125m-block"]
    data = make_inputs(wl)
    X = data["X"]["attn_in"].cuda()
    Ls = [L for L in wl.layers if L.input_name == "attn_in"]
    Ws = [data["W"][L.name].cuda() for L in Ls]
    ctr = ttq.new_counter()
    sums, s, inv = ttq.act_stats_scales(X, ctr, wl.alpha, wl.lam, wl.p)
    Xs, _ = ttq.prepare_activations(X, inv, wl.bits)
    cs, ds, zs = ttq.quantize_rtn_grouped(torch.cat(Ws), s, wl.bits, wl.group)
    Ys = ttq.w_lowbit_gemm_prepared(Xs, None, cs, ds, zs, cs.shape[0], wl.bits,
                                    wl.group, out_dtype=wl.dtype)
    row = 0
    for L, W in zip(Ls, Ws):
        c, d, z = ttq.quantize_rtn_grouped(W, s, wl.bits, wl.group)
        assert torch.equal(c, cs[row:row + L.N])
        assert torch.equal(d, ds[row:row + L.N])
        assert torch.equal(z, zs[row:row + L.N])
        Y = ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, L.N, wl.bits,
                                       wl.group, out_dtype=wl.dtype)
        # same operands, same K order: the tensor-core sums agree exactly
        assert torch.equal(Y, Ys[:, row:row + L.N])
        row += L.N
    tok = sample_rows(wl.T, 8, 5)
    cd, dd, zd = dense(cs, ds, zs, X.shape[1], wl.bits, wl.group)
    ref = oracle.lowbit_gemm(np32(X.cpu()[:wl.T]), np32(inv), cd, dd, zd,
                             cs.shape[0], wl.bits, wl.group, rows=tok)
    assert_gemm_close(np32(Ys)[tok], ref, "stacked q|k|v", Ys.dtype)
    assert int(ctr.item()) == 0
