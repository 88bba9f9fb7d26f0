"""Pins of the CPU oracle to facts fixed by the pages and by mathematics.

None of these tests retypes an oracle formula: each checks the oracle against
a closed form, a special case that reduces to a library routine, a
brute-force search, an invariant, or a hand-worked example (tests/golden).
Source of the method: TTQ review (nubint.ai), section "Proposed method",
bullets 1-5.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- stats ---

@pytest.mark.parametrize("p", [1.0, 2.0, 3.0])
def test_stats_constant_input_closed_form(p):
    T, K = 37, 64
    a = -1.5
    X = np.full((T, K), a, np.float32)
    sums = oracle.act_sums(X, p)
    np.testing.assert_allclose(sums, T * abs(a) ** p, rtol=1e-14)


def test_stats_one_hot_rows():
    rng = np.random.default_rng(1)
    T, K = 50, 96
    cols = rng.integers(0, K, T)
    vals = rng.standard_normal(T).astype(np.float32)
    X = np.zeros((T, K), np.float32)
    X[np.arange(T), cols] = vals
    sums = oracle.act_sums(X, 2.0)
    expect = np.zeros(K)
    for c, v in zip(cols, vals):
        expect[c] += float(v) ** 2
    np.testing.assert_allclose(sums, expect, rtol=1e-13, atol=0)


def test_stats_sign_permutation_and_chunking():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((80, 64)).astype(np.float32)
    for p in (1.0, 2.0, 3.0):
        full = oracle.act_sums(X, p)
        np.testing.assert_allclose(oracle.act_sums(-X, p), full, rtol=1e-13)
        perm = rng.permutation(80)
        np.testing.assert_allclose(oracle.act_sums(X[perm], p), full,
                                   rtol=1e-12)
        chunked = oracle.act_sums(X[:33], p) + oracle.act_sums(X[33:], p)
        np.testing.assert_allclose(chunked, full, rtol=1e-12)


# ---------------------------------------------------------------- scales ---

def _sums(seed=3, T=64, K=48):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, K)).astype(np.float32)
    X[:, 5] *= 20
    return oracle.act_sums(X, 2.0), T


def test_scales_alpha_zero_is_plain_rtn_scale():
    sums, T = _sums()
    s, inv = oracle.awq_scales(sums, T, 0.0, 0.1, 2.0)
    assert np.all(s == 1.0) and np.all(inv == 1.0)


def test_scales_alpha_equals_p_without_shrink_is_the_statistic():
    # c^(alpha/p) with alpha = p is c itself, and lambda = 0 leaves c = m.
    sums, T = _sums()
    s, _ = oracle.awq_scales(sums, T, 2.0, 0.0, 2.0)
    np.testing.assert_allclose(s, sums / T, rtol=1e-15)


def test_scales_full_shrink_is_the_mean_statistic():
    sums, T = _sums()
    s, _ = oracle.awq_scales(sums, T, 2.0, 1.0, 2.0)
    np.testing.assert_allclose(s, np.full_like(s, np.mean(sums / T)),
                               rtol=1e-13)


def test_scales_shrink_is_affine_in_lambda():
    # With alpha = p the scale equals c, which must be the midpoint of the
    # lambda = 0 and lambda = 1 cases at lambda = 1/2 (a convex shrink).
    sums, T = _sums()
    s0, _ = oracle.awq_scales(sums, T, 2.0, 0.0, 2.0)
    s1, _ = oracle.awq_scales(sums, T, 2.0, 1.0, 2.0)
    sh, _ = oracle.awq_scales(sums, T, 2.0, 0.5, 2.0)
    np.testing.assert_allclose(sh, 0.5 * (s0 + s1), rtol=1e-13)


@pytest.mark.parametrize("alpha,lam,p", [(0.5, 0.1, 2.0), (0.3, 0.0, 1.0),
                                         (0.8, 0.5, 2.0)])
def test_scales_homogeneity(alpha, lam, p):
    # Scaling X by a multiplies every p-th moment by |a|^p, so s by |a|^alpha.
    rng = np.random.default_rng(4)
    X = rng.standard_normal((40, 32)).astype(np.float32)
    a = 4.0
    s1, inv1 = oracle.awq_scales(oracle.act_sums(X, p), 40, alpha, lam, p)
    s2, _ = oracle.awq_scales(oracle.act_sums(a * X, p), 40, alpha, lam, p)
    np.testing.assert_allclose(s2 / s1, a ** alpha, rtol=1e-12)
    np.testing.assert_allclose(s1 * inv1, 1.0, rtol=1e-15)


def test_scales_monotone_in_statistic():
    sums, T = _sums()
    s, _ = oracle.awq_scales(sums, T, 0.5, 0.1, 2.0)
    order = np.argsort(sums)
    assert np.all(np.diff(s[order]) >= 0)


def test_scales_degenerate_zero_statistic():
    s, inv = oracle.awq_scales(np.zeros(32), 10, 0.5, 0.0, 2.0)
    assert np.all(s == 1.0) and np.all(inv == 1.0)


# -------------------------------------------------------------- quantize ---

def _golden_cases():
    with open(os.path.join(GOLDEN, "quantize_handworked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_quantize_hand_worked(case):
    W = np.array(case["W"], np.float32)
    s = None if case["s"] is None else np.array(case["s"], np.float32)
    codes, delta, zero = oracle.quantize(W, s, case["bits"], case["group"])
    q = oracle.unpack_codes(codes, case["K"], case["bits"])
    np.testing.assert_array_equal(q, np.array(case["q"], np.uint8))
    np.testing.assert_array_equal(delta, np.array(case["delta"], np.float32))
    np.testing.assert_array_equal(zero, np.array(case["zero"], np.uint8))
    words = np.array([[int(h, 16) for h in row] for row in case["codes_hex"]],
                     np.uint32)
    np.testing.assert_array_equal(codes, words)


def _bitstream_pack(q_row, bits):
    """Independent packing: one Python integer per 32-code block."""
    out = []
    for b0 in range(0, len(q_row), 32):
        v = 0
        for c, qc in enumerate(q_row[b0:b0 + 32]):
            v |= int(qc) << (c * bits)
        out += [(v >> (32 * w)) & 0xFFFFFFFF for w in range(bits)]
    return out


@pytest.mark.parametrize("bits", range(2, 9))
def test_pack_matches_bitstream_and_round_trips(bits):
    rng = np.random.default_rng(bits)
    q = rng.integers(0, 1 << bits, (3, 96)).astype(np.uint8)
    codes = oracle.pack_codes(q, bits)
    for n in range(3):
        assert list(codes[n]) == _bitstream_pack(q[n], bits)
    np.testing.assert_array_equal(oracle.unpack_codes(codes, 96, bits), q)


@pytest.mark.parametrize("bits", range(2, 9))
@pytest.mark.parametrize("group", [16, 32])
def test_quantize_brute_force_argmin(bits, group):
    """Every code is the nearest grid point among all 2^b (tiny inputs)."""
    rng = np.random.default_rng(100 * bits + group)
    N, K = 4, 64
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s = np.exp(rng.standard_normal(K) * 0.5).astype(np.float32)
    codes, delta, zero = oracle.quantize(W, s, bits, group)
    q = oracle.unpack_codes(codes, K, bits)
    qmax = (1 << bits) - 1
    grid = np.arange(qmax + 1, dtype=np.float64)
    checked = 0
    for n in range(N):
        for j in range(K):
            g = j // group
            d = float(delta[n, g])
            z = float(zero[n, g])
            w = float(np.float32(W[n, j]) * np.float32(s[j]))
            err = np.abs(w - (grid - z) * d)
            best = np.sort(err)
            if best[1] - best[0] < 1e-6 * d:   # near-tie: either is nearest
                continue
            assert q[n, j] == int(np.argmin(err)), (n, j)
            checked += 1
    assert checked > 0.95 * N * K


def test_quantize_grid_properties_and_error_bound():
    rng = np.random.default_rng(7)
    N, K = 16, 256
    for bits in (2, 3, 4, 5, 8):
        for group in (16, 32, 64, 128):
            W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
            s = np.exp(rng.standard_normal(K)).astype(np.float32)
            codes, delta, zero = oracle.quantize(W, s, bits, group)
            What = oracle.dequantize(codes, delta, zero, K, bits, group)
            Ws = (W * s[None, :]).astype(np.float64)   # fp32 product, exact
            D = np.repeat(delta.astype(np.float64), group, axis=1)
            assert np.all(np.abs(What - Ws) <= D / 2 * (1 + 2 ** -20))
            qmax = (1 << bits) - 1
            wg = Ws.reshape(N, K // group, group)
            mn = np.minimum(wg.min(axis=2), 0)
            mx = np.maximum(wg.max(axis=2), 0)
            # the step is the range split into 2^b - 1 intervals
            np.testing.assert_allclose(delta, (mx - mn) / qmax, rtol=2e-7)
            # zero is representable exactly: q == z reconstructs 0
            assert np.all(zero <= qmax)


def test_quantize_power_of_two_scale_invariance():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((8, 128)) * 0.02).astype(np.float32)
    s = np.exp(rng.standard_normal(128)).astype(np.float32)
    c1, d1, z1 = oracle.quantize(W, s, 4, 32)
    c2, d2, z2 = oracle.quantize(W, s * np.float32(8.0), 4, 32)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(z1, z2)
    np.testing.assert_array_equal(d2, d1 * np.float32(8.0))


def test_quantize_exact_grid_weights_reconstruct_exactly():
    rng = np.random.default_rng(9)
    bits, group, N, K = 4, 32, 6, 128
    qmax = (1 << bits) - 1
    q = rng.integers(0, qmax + 1, (N, K))
    z = rng.integers(1, qmax, (N, K // group))
    # make every group reach both ends of the grid
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    d = 2.0 ** -rng.integers(3, 8, (N, K // group))
    W = ((q - np.repeat(z, group, 1)) * np.repeat(d, group, 1)).astype(
        np.float32)
    codes, delta, zero = oracle.quantize(W, None, bits, group)
    np.testing.assert_array_equal(oracle.unpack_codes(codes, K, bits), q)
    np.testing.assert_array_equal(zero, z)
    np.testing.assert_array_equal(delta, d.astype(np.float32))


def test_quantize_error_shrinks_with_bits_and_vanishes_at_8_bits():
    # Large b with g = K drives W_hat toward W (bound D/2 = range/(2(2^b-1))).
    rng = np.random.default_rng(10)
    K = 128
    W = (rng.standard_normal((8, K)) * 0.02).astype(np.float32)
    errs = []
    for bits in range(2, 9):
        c, d, z = oracle.quantize(W, None, bits, K)
        errs.append(np.max(np.abs(oracle.dequantize(c, d, z, K, bits, K) - W)))
    assert all(b < a for a, b in zip(errs, errs[1:]))
    rng_w = float(W.max() - min(W.min(), 0) if W.min() < 0 else W.max())
    assert errs[-1] <= rng_w / 255 / 2 * (1 + 1e-6) + 1e-12


def test_quantize_one_signed_and_zero_groups():
    W = np.zeros((3, 32), np.float32)
    W[1, :16] = np.linspace(0.1, 1.0, 16)
    W[2, :16] = -np.linspace(0.1, 1.0, 16)
    codes, delta, zero = oracle.quantize(W, None, 3, 16)
    q = oracle.unpack_codes(codes, 32, 3)
    assert delta[0, 0] == 1.0 and zero[0, 0] == 0 and np.all(q[0] == 0)
    assert zero[1, 0] == 0 and q[1, 15] == 7
    assert zero[2, 0] == 7 and q[2, 15] == 0


# ------------------------------------------------------------------ gemm ---

def _quantized_layer(seed, T=24, N=40, K=96, bits=3, group=32, r=0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, K)).astype(np.float32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s, inv = oracle.awq_scales(oracle.act_sums(X), T, 0.5, 0.1, 2.0)
    codes, delta, zero = oracle.quantize(W, s, bits, group)
    A = B = None
    if r:
        A = rng.standard_normal((r, K)).astype(np.float32) * 0.1
        B = rng.standard_normal((N, r)).astype(np.float32) * 0.1
    return X, W, s.astype(np.float32), inv.astype(np.float32), codes, delta, \
        zero, A, B


@pytest.mark.parametrize("r", [0, 4])
def test_gemm_equals_dense_matmul_of_dequantized_weight(r):
    X, W, s, inv, codes, delta, zero, A, B = _quantized_layer(11, r=r)
    N, K = W.shape
    Y = oracle.lowbit_gemm(X, inv, codes, delta, zero, N, 3, 32, A, B)
    What = oracle.dequantize(codes, delta, zero, K, 3, 32)
    ref = (X.astype(np.float64) * inv.astype(np.float64)) @ What.T
    if r:
        ref = ref + (X.astype(np.float64) @ A.astype(np.float64).T) @ \
            B.astype(np.float64).T
    np.testing.assert_allclose(Y, ref, rtol=1e-11, atol=1e-13)
    rows = [3, 0, 17]
    np.testing.assert_allclose(
        oracle.lowbit_gemm(X, inv, codes, delta, zero, N, 3, 32, A, B,
                           rows=rows), Y[rows], rtol=0, atol=0)


def test_gemm_one_hot_token_picks_a_weight_column():
    X, W, s, inv, codes, delta, zero, _, _ = _quantized_layer(12)
    N, K = W.shape
    Xo = np.zeros((1, K), np.float32)
    Xo[0, 7] = 1.0
    Y = oracle.lowbit_gemm(Xo, inv, codes, delta, zero, N, 3, 32)
    q = oracle.unpack_codes(codes, K, 3)[:, 7].astype(np.float64)
    col = (q - zero[:, 0]) * delta[:, 0].astype(np.float64) * float(inv[7])
    np.testing.assert_allclose(Y[0], col, rtol=1e-15)


def test_gemm_exact_grid_weights_give_plain_projection():
    rng = np.random.default_rng(13)
    bits, group, N, K, T = 4, 32, 8, 64, 5
    qmax = (1 << bits) - 1
    q = rng.integers(0, qmax + 1, (N, K))
    q[:, ::group] = 0
    q[:, 1::group] = qmax
    z = rng.integers(1, qmax, (N, K // group))
    d = 2.0 ** -rng.integers(3, 8, (N, K // group))
    W = ((q - np.repeat(z, group, 1)) * np.repeat(d, group, 1)).astype(
        np.float32)
    X = rng.standard_normal((T, K)).astype(np.float32)
    codes, delta, zero = oracle.quantize(W, None, bits, group)
    Y = oracle.lowbit_gemm(X, np.ones(K, np.float32), codes, delta, zero, N,
                           bits, group)
    np.testing.assert_allclose(Y, X.astype(np.float64) @ W.T.astype(
        np.float64), rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------ loss ---

def test_loss_zero_for_exact_weight_and_trace_form():
    rng = np.random.default_rng(14)
    T, N, K = 30, 12, 64
    X = rng.standard_normal((T, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32)
    assert oracle.loss(W, W.astype(np.float64), X) == 0.0
    We = W.astype(np.float64) + rng.standard_normal((N, K)) * 1e-3
    E = W.astype(np.float64) - We
    C = X.astype(np.float64).T @ X.astype(np.float64) / T
    np.testing.assert_allclose(oracle.loss(W, We, X), np.trace(E @ C @ E.T),
                               rtol=1e-10)


@pytest.mark.parametrize("seed", [20, 21, 22])
def test_ttq_loss_not_above_rtn_on_outlier_inputs(seed):
    """Activation-aware scales reduce E||(W - W_hat) x||^2 when a few input
    channels carry outliers (Proposed method, bullets 2-3; Main results,
    bullet 1). Asserted on these fixed seeds, not as a theorem."""
    rng = np.random.default_rng(seed)
    T, N, K = 128, 64, 256
    X = rng.standard_normal((T, K)).astype(np.float32)
    X[:, rng.choice(K, 8, replace=False)] *= 20
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s, _ = oracle.awq_scales(oracle.act_sums(X), T, 0.5, 0.1, 2.0)
    s32 = s.astype(np.float32)
    c, d, z = oracle.quantize(W, s32, 4, 32)
    l_ttq = oracle.loss(W, oracle.effective_weight(c, d, z, s32, K, 4, 32), X)
    c0, d0, z0 = oracle.quantize(W, None, 4, 32)
    l_rtn = oracle.loss(W, oracle.effective_weight(c0, d0, z0, None, K, 4, 32),
                        X)
    assert l_ttq <= l_rtn


# -------------------------------------------------------------- low rank ---

def test_lowrank_residual_reconstructs_weight():
    """W_q + B A reconstructs W within the quantizer's bound (bullet 5)."""
    from test_weight_quantization_b200.inputs import lowrank_checkpoint
    rng = np.random.default_rng(15)
    N, K, r = 48, 128, 16
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    R, A, B = lowrank_checkpoint(W, r)
    Rf, Af, Bf = (t.float().numpy() for t in (R, A, B))
    c, d, z = oracle.quantize(Rf, None, 4, 32)
    Rq = oracle.dequantize(c, d, z, K, 4, 32)
    recon = Rq + Bf.astype(np.float64) @ Af.astype(np.float64)
    bound = np.repeat(d.astype(np.float64), 32, 1) / 2 * (1 + 2 ** -20)
    # bf16 storage of the residual adds at most half a bf16 ulp of R
    bound = bound + np.abs(Rf) * 2 ** -8
    assert np.all(np.abs(recon - W) <= bound + 1e-7)
    # the rank-r part carries the top singular directions: the residual is
    # smaller than W in Frobenius norm
    assert np.linalg.norm(Rf) < np.linalg.norm(W)


def test_near_tie_counter_sees_exact_ties():
    W = np.zeros((1, 32), np.float32)
    W[0, :4] = [-1.0, 2.0, 0.5, 1.5]      # D = 1: 0.5 and 1.5 are ties
    assert oracle.count_near_ties(W, None, 2, 16) >= 2
