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
from fractions import Fraction

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


def test_scales_of_channel_shards_with_the_global_mean_equal_the_whole():
    """Splitting the channels into shards and giving every shard the mean
    over all channels reproduces the scales of the unsplit layer; giving it
    its own shard's mean does not (the shrinkage mixes in all channels)."""
    rng = np.random.default_rng(21)
    T, K = 40, 96
    X = rng.standard_normal((T, K)) * np.exp(rng.standard_normal(K))
    sums = oracle.act_sums(X)
    s, inv = oracle.awq_scales(sums, T, 0.5, 0.3, 2.0)
    mbar = float(np.mean(sums / T))
    parts = [oracle.awq_scales_given_mean(sums[a:b], T, mbar, 0.5, 0.3, 2.0)
             for a, b in ((0, 32), (32, 96))]
    np.testing.assert_allclose(np.concatenate([p[0] for p in parts]), s,
                               rtol=1e-13)
    np.testing.assert_allclose(np.concatenate([p[1] for p in parts]), inv,
                               rtol=1e-13)
    own, _ = oracle.awq_scales_given_mean(sums[:32], T,
                                          float(np.mean(sums[:32] / T)), 0.5,
                                          0.3, 2.0)
    assert np.max(np.abs(own / s[:32] - 1)) > 1e-3


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


# ------------------------------------------- RTN by its exact definition ---
# Group RTN divides: q = rint(w/D) + z and z = rint(-mn/D), each quotient
# one IEEE fp32 division (correctly rounded) and rint round-half-to-even.
# The references below evaluate that definition in exact rational
# arithmetic, rounding to fp32 by hand, so they share no floating-point
# operation with the oracle.

def _rn32(x: Fraction) -> float:
    """x rounded to the nearest fp32 value, ties to even."""
    if x == 0:
        return 0.0
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    step = Fraction(2) ** (max(e, -126) - 23)
    m = a / step
    f = m.numerator // m.denominator
    rem = m - f
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and f % 2 == 1):
        f += 1
    return math.copysign(float(f * step), float(x))


def _exact_rtn_group(w, bits):
    """(codes, D, z) of one group of fp32 scaled weights, exactly."""
    qmax = (1 << bits) - 1
    mn = min(0.0, float(w.min()))
    mx = max(0.0, float(w.max()))
    d = _rn32(Fraction(_rn32(Fraction(mx) - Fraction(mn))) / qmax)
    if d == 0.0:
        d = 1.0
    z = min(max(round(_rn32(Fraction(-mn) / Fraction(d))), 0), qmax)
    q = [min(max(round(_rn32(Fraction(float(v)) / Fraction(d))) + z, 0), qmax)
         for v in w]
    return q, d, z


def _reciprocal_disagreements(seed, bits, count):
    """Groups where rint(x * (1/D)) and rint(x / D) differ, found by a
    seeded search over random (min, max, weight) triples in numpy fp32:
    rows of 32 weights [mn, mx, w, 0, ...] whose first group's zero point
    or third weight rounds differently under the two."""
    rng = np.random.default_rng(seed)
    M = 1 << 22
    qmax = np.float32((1 << bits) - 1)
    mn = -np.abs(rng.standard_normal(M)).astype(np.float32)
    mx = np.abs(rng.standard_normal(M)).astype(np.float32)
    w = (rng.uniform(-1, 1, M).astype(np.float32) *
         np.maximum(-mn, mx)).astype(np.float32)
    w = np.clip(w, mn, mx)
    d = (mx - mn) / qmax
    r = np.float32(1) / d
    zero_idx = np.nonzero(np.rint(-mn / d) != np.rint(-mn * r))[0][:count]
    weight_idx = np.nonzero(np.rint(w / d) != np.rint(w * r))[0][:count]
    rows = []
    for i in np.concatenate([zero_idx, weight_idx]):
        row = np.zeros(32, np.float32)   # a second, all-zero group
        row[:3] = [mn[i], mx[i], w[i]]
        rows.append(row)
    return np.array(rows, np.float32), len(zero_idx), len(weight_idx)


@pytest.mark.parametrize("bits,seed", [(8, 40), (7, 41)])
def test_quantize_is_rtn_by_division_not_by_reciprocal(bits, seed):
    """On groups where a rounded reciprocal would change the zero point or a
    code, the oracle gives the exact rounding of the quotients. (Such groups
    are rarer at fewer bits, where the quotients are smaller.)"""
    W, n_zero, n_weight = _reciprocal_disagreements(seed, bits, 12)
    assert n_zero >= 3 and n_weight >= 3, (n_zero, n_weight)
    codes, delta, zero = oracle.quantize(W, None, bits, 16)
    q = oracle.unpack_codes(codes, 32, bits)
    for n in range(W.shape[0]):
        eq, ed, ez = _exact_rtn_group(W[n, :16], bits)
        assert float(delta[n, 0]) == ed, n
        assert int(zero[n, 0]) == ez, n
        assert list(q[n, :16]) == eq, n


def test_quantize_matches_exact_definition_on_random_groups():
    rng = np.random.default_rng(12)
    for bits, group in ((2, 16), (3, 32), (5, 64), (8, 128)):
        W = (rng.standard_normal((3, 256)) * 0.02).astype(np.float32)
        s = np.exp(rng.standard_normal(256) * 0.6).astype(np.float32)
        codes, delta, zero = oracle.quantize(W, s, bits, group)
        q = oracle.unpack_codes(codes, 256, bits)
        Ws = W * s[None, :]
        for n in range(3):
            for gi in range(256 // group):
                sl = slice(gi * group, (gi + 1) * group)
                eq, ed, ez = _exact_rtn_group(Ws[n, sl], bits)
                assert float(delta[n, gi]) == ed
                assert int(zero[n, gi]) == ez
                assert list(q[n, sl]) == eq


def _steps_from(v, k):
    """The fp32 value k representable steps from v (k may be negative)."""
    out = np.float32(v)
    for _ in range(abs(k)):
        out = np.nextafter(out, np.float32(np.inf if k > 0 else -np.inf),
                           dtype=np.float32)
    return out


def test_near_tie_mask_is_one_step_wide():
    """D = 1 exactly (b = 4, range [0, 15]), so each quotient is the weight
    itself: the tie and its two neighbours count, two and three steps away
    do not."""
    W = np.zeros((1, 16), np.float32)
    W[0, 0] = 15.0
    offsets = [0, 1, -1, 2, -2, 3]
    for i, k in enumerate(offsets):
        W[0, 1 + i] = _steps_from(2.5, k)
    W[0, 7] = 3.0
    _, delta, _ = oracle.quantize(W, None, 4, 16)
    assert delta[0, 0] == 1.0
    mask, weights, groups = oracle.near_tie_mask(W, None, 4, 16)
    assert list(mask[0, 1:7]) == [1, 1, 1, 0, 0, 0]
    assert mask[0, 0] == 0 and mask[0, 7] == 0
    assert weights == 3 and groups == 0
    assert oracle.count_near_ties(W, None, 4, 16) == 3


def test_near_tie_mask_counts_zero_point_groups():
    """Three groups with D = 1 (b = 4) whose zero-point quotient -mn/D is
    2.5 exactly, one step above it, and three steps above it: the first two
    are zero-point near-ties and every weight of theirs is marked."""
    mns = [np.float32(-2.5), -_steps_from(2.5, 1), -_steps_from(2.5, 3)]
    mxs = [np.float32(12.5), np.float32(12.5),
           np.float32(12.5) - np.float32(2.0 ** -20)]
    W = np.zeros((3, 16), np.float32)
    W[:, 3:] = 1.0
    for n in range(3):
        W[n, 0], W[n, 1] = mns[n], mxs[n]
    _, delta, zero = oracle.quantize(W, None, 4, 16)
    assert np.all(delta == 1.0)
    # the construction: quotients 2.5, one step and three steps above it
    assert [int(np.round((-W[n, 0] - np.float32(2.5)) /
                         np.float32(2.0 ** -22))) for n in range(3)] == \
        [0, 1, 3]
    mask, weights, groups = oracle.near_tie_mask(W, None, 4, 16)
    assert groups == 2
    assert np.all(mask[:2] != 0)          # whole groups excused
    # mn and mx are themselves weights within a step of -2.5 and 12.5
    assert list(mask[0, :2]) == [3, 3] and list(mask[1, :2]) == [3, 3]
    assert np.all(mask[:2, 2:] == 2)
    assert mask[2, 1] == 1 and mask[2, 0] == 0 and np.all(mask[2, 2:] == 0)
    assert weights == 5
