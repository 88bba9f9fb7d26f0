"""GPU parity: every step of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs.

Small shapes span several tiles and a ragged tail; the oracle is always fed
the GPU's own upstream outputs (sums -> scales -> codes) so each step is
compared on identical inputs. Tolerances: see parity_util.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_codes_match, assert_gemm_close,
                         assert_rel_close, gemm_errors, np32)

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@pytest.fixture(scope="module")
def ttq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_weight_quantization_b200 import ttq as mod
    mod.device_error(clear=True)
    yield mod
    assert mod.device_error(clear=True) == 0


def acts(T, K, seed, dtype, frac=0.02, factor=20.0):
    from test_weight_quantization_b200.inputs import activations
    X = activations(T, K, seed, "student_t", outlier_frac=frac,
                    outlier_factor=factor)
    return torch.from_numpy(X).to(dtype)


def weights(N, K, seed, dtype):
    from test_weight_quantization_b200.inputs import weights as w
    return torch.from_numpy(w(N, K, seed)).to(dtype)


# ------------------------------------------------------------- stats ----

@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("T,K", [(1, 8), (37, 264), (300, 1000), (1000, 2056)])
@pytest.mark.parametrize("p", [2.0, 1.0, 3.0])
def test_stats(ttq, dt, T, K, p):
    X = acts(T, K, T + K, DT[dt])
    got = ttq.act_stats(X.cuda(), p)
    ref = oracle.act_sums(np32(X), p)
    assert_rel_close(np32(got), ref, what="sums")


def test_stats_accumulate_and_pitch(ttq):
    X = acts(700, 512, 5, torch.bfloat16)
    big = torch.zeros(700, 640, dtype=torch.bfloat16)
    big[:, :512] = X
    Xg = big.cuda()[:, :512]  # row pitch 640
    out = ttq.act_stats(Xg[:300])
    ttq.act_stats(Xg[300:], out=out, accumulate=True)
    assert_rel_close(np32(out), oracle.act_sums(np32(X)), what="chunked")


def test_stats_deterministic(ttq):
    Xg = acts(2048, 768, 6, torch.bfloat16).cuda()
    a = ttq.act_stats(Xg)
    b = ttq.act_stats(Xg)
    assert torch.equal(a, b)


# ------------------------------------------------------------ scales ----

@pytest.mark.parametrize("alpha,lam,p", [(0.5, 0.1, 2.0), (0.0, 0.1, 2.0),
                                         (0.7, 1.0, 2.0), (0.4, 0.0, 1.0)])
def test_scales(ttq, alpha, lam, p):
    X = acts(512, 1024, 7, torch.bfloat16)
    sums = ttq.act_stats(X.cuda(), p)
    s, inv = ttq.awq_scales(sums, 512, alpha, lam, p)
    rs, rinv = oracle.awq_scales(np32(sums).astype(np.float64), 512, alpha,
                                 lam, p)
    assert_rel_close(np32(s), rs, what="s")
    assert_rel_close(np32(inv), rinv, what="inv_s")


def test_scales_zero_statistic(ttq):
    sums = torch.zeros(256, device="cuda")
    s, inv = ttq.awq_scales(sums, 10, 0.5, 0.0, 2.0)
    assert torch.all(s == 1) and torch.all(inv == 1)


# ------------------------------------------------ fused stats + scales ----

@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("T,K", [(1, 8), (37, 264), (2048, 768),
                                 (300, 3072), (64, 14336)])
@pytest.mark.parametrize("alpha,lam,p", [(0.5, 0.1, 2.0), (0.0, 0.1, 2.0),
                                         (0.4, 0.0, 1.0), (0.6, 0.3, 3.0)])
def test_stats_scales_fused(ttq, dt, T, K, alpha, lam, p):
    """One launch gives the sums of act_stats bit for bit and the oracle's
    scales; the counter comes back to zero."""
    X = acts(T, K, 3 * T + K, DT[dt]).cuda()
    ctr = ttq.new_counter()
    sums, s, inv = ttq.act_stats_scales(X, ctr, alpha, lam, p)
    assert torch.equal(sums, ttq.act_stats(X, p))
    rs, rinv = oracle.awq_scales(np32(sums).astype(np.float64), T, alpha, lam,
                                 p)
    assert_rel_close(np32(s), rs, what="fused s")
    assert_rel_close(np32(inv), rinv, what="fused inv_s")
    s2, inv2 = ttq.awq_scales(sums, T, alpha, lam, p)
    assert torch.allclose(s, s2, rtol=1e-6, atol=0)
    assert int(ctr.item()) == 0


def test_stats_scales_fused_repeated_and_accumulate(ttq):
    """Back-to-back calls reuse one counter; the chunked form divides by the
    running token count."""
    X = acts(900, 1152, 11, torch.bfloat16).cuda()
    ctr = ttq.new_counter()
    first = [t.clone() for t in ttq.act_stats_scales(X, ctr)]
    for _ in range(5):
        again = ttq.act_stats_scales(X, ctr)
        for a, b in zip(first, again):
            assert torch.equal(a, b)
    sums, s, inv = ttq.act_stats_scales(X[:400], ctr)
    sums, s, inv = ttq.act_stats_scales(X[400:], ctr, sums=sums, s=s,
                                        inv_s=inv, accumulate=True,
                                        T_total=900)
    assert_rel_close(np32(sums), oracle.act_sums(np32(X.cpu())),
                     what="chunked sums")
    rs, rinv = oracle.awq_scales(np32(sums).astype(np.float64), 900, 0.5, 0.1,
                                 2.0)
    assert_rel_close(np32(s), rs, what="chunked s")
    assert int(ctr.item()) == 0


def test_stats_scales_fused_zero_input(ttq):
    X = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    ctr = ttq.new_counter()
    sums, s, inv = ttq.act_stats_scales(X, ctr, 0.5, 0.0, 2.0)
    assert torch.all(sums == 0) and torch.all(s == 1) and torch.all(inv == 1)


# ------------------------------------------- sharded (row-parallel) scales ----

def test_channel_total_and_sharded_scales(ttq):
    """Input channels split in two shards: each shard's channel total, added
    (the all-reduce of a row-parallel layer, here on one GPU), gives every
    shard the scales the unsplit layer has."""
    T, K = 300, 1152
    X = acts(T, K, 71, torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s_full, inv_full = ttq.awq_scales(sums, T, 0.5, 0.1, 2.0)
    parts, totals = [], []
    for a, b in ((0, 512), (512, 1152)):
        sh = ttq.act_stats(X[:, a:b].contiguous())
        parts.append(sh)
        totals.append(ttq.channel_moment_total(sh, T))
    total = totals[0] + totals[1]
    # each shard's total is the fp64 sum of its own channel sums (which
    # differ from the unsplit statistics' in the last fp32 bits: another
    # accumulation order)
    ref_total = sum(np.sum(np32(sh).astype(np.float64) / T) for sh in parts)
    assert abs(total.item() - ref_total) <= 1e-12 * abs(ref_total)
    got = [ttq.awq_scales_sharded(sh, T, K, total, 0.5, 0.1, 2.0)
           for sh in parts]
    s = torch.cat([g[0] for g in got])
    inv = torch.cat([g[1] for g in got])
    rs, rinv = oracle.awq_scales(np32(sums).astype(np.float64), T, 0.5, 0.1,
                                 2.0)
    assert_rel_close(np32(s), rs, what="sharded s")
    assert_rel_close(np32(inv), rinv, what="sharded inv_s")
    assert torch.allclose(s, s_full, rtol=1e-6, atol=0)


def test_row_parallel_projection_on_one_gpu(ttq):
    """The row-parallel layer's arithmetic, its two ranks run one after the
    other on one GPU and their fp32 partial outputs added: the oracle's
    unsplit projection within the projection tolerance."""
    T, N, K, bits, group = 200, 320, 1024, 4, 128
    X = acts(T, K, 72, torch.bfloat16).cuda()
    W = weights(N, K, 73, torch.bfloat16).cuda()
    shards = ((0, 512), (512, 1024))
    sums = [ttq.act_stats(X[:, a:b].contiguous()) for a, b in shards]
    total = sum(ttq.channel_moment_total(sh, T) for sh in sums)
    Y = torch.zeros(T, N, dtype=torch.float32, device="cuda")
    for (a, b), sh in zip(shards, sums):
        s, inv = ttq.awq_scales_sharded(sh, T, K, total)
        c, d, z = ttq.quantize_rtn_grouped(W[:, a:b].contiguous(), s, bits,
                                           group)
        Y += ttq.w_lowbit_gemm(X[:, a:b].contiguous(), inv, c, d, z, N, bits,
                               group, out_dtype=torch.float32)
    # the oracle's unsplit layer on the GPU's scales
    s_full, inv_full = ttq.awq_scales(ttq.act_stats(X), T)
    c, d, z = ttq.quantize_rtn_grouped(W, s_full, bits, group)
    ref = oracle_y(X.cpu(), inv_full, c, d, z, N, bits, group)
    assert_gemm_close(np32(Y), ref, "row-parallel on one GPU", Y.dtype)


# ------------------------------- quantization fused into the projection ----

@pytest.mark.parametrize("bits,group", [(4, 128), (3, 32), (2, 16), (5, 64),
                                        (8, 128), (4, 64), (6, 16)])
@pytest.mark.parametrize("T,N,K", [(300, 272, 1152), (64, 130, 1056)])
def test_fused_quantize_projection_equals_two_passes(ttq, bits, group, T, N,
                                                     K):
    """The projection that quantizes the bf16 weights itself gives the two-
    pass result (quantize, then project) bit for bit, and stores the same
    codes, delta and zero; several token tiles, ragged N, a K whose last
    128-channel stage is partial, every group size (64 and 128 span several
    dequantiser warps)."""
    if K % group:
        pytest.skip("K not a multiple of g")
    X = acts(T, K, 100 + bits, torch.bfloat16).cuda()
    W = weights(N, K, 101 + group, torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s, inv = ttq.awq_scales(sums, T)
    Xs, _ = ttq.prepare_activations(X, inv, bits)
    c, d, z = ttq.quantize_rtn_grouped(W, s, bits, group)
    ref = ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, N, bits, group)
    Y, (fc, fd, fz) = ttq.quantize_gemm_prepared(W, s, Xs, None, bits, group)
    torch.cuda.synchronize()
    w, G = K * bits // 32, K // group
    assert torch.equal(fc[:, :w], c[:, :w])
    assert torch.equal(fd[:, :G], d[:, :G])
    assert torch.equal(fz[:, :G], z[:, :G])
    Y2, none = ttq.quantize_gemm_prepared(W, s, Xs, None, bits, group,
                                          store_codes=False)
    assert none is None and torch.equal(Y2, Y)
    if T > 256:
        # several token tiles: the same tiles in the same order, bit for bit
        assert torch.equal(Y, ref)
    else:
        # one token tile: the fused form splits K over a cluster, so the
        # fp32 sums run in another order; against the oracle's projection
        ref_o = oracle_y(X.cpu(), inv.cpu(), c.cpu(), d.cpu(), z.cpu(), N,
                         bits, group)
        assert_gemm_close(np32(Y), ref_o, "fused, K split", Y.dtype)
        assert_gemm_close(np32(ref), ref_o, "two passes", ref.dtype)


def test_fused_quantize_projection_lowrank_and_oracle(ttq):
    """With the low-rank stage, against the oracle's projection."""
    T, N, K, r, bits, group = 200, 272, 384, 16, 4, 64
    X = acts(T, K, 110, torch.bfloat16)
    W = weights(N, K, 111, torch.bfloat16)
    rng = np.random.default_rng(112)
    A = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32) * .05
                         ).to(torch.bfloat16).cuda()
    B = torch.from_numpy(rng.standard_normal((N, r)).astype(np.float32) * .05
                         ).to(torch.bfloat16).cuda()
    Xg, Wg = X.cuda(), W.cuda()
    s, inv = ttq.awq_scales(ttq.act_stats(Xg), T)
    Xs, U = ttq.prepare_activations(Xg, inv, bits, A)
    Y, (c, d, z) = ttq.quantize_gemm_prepared(Wg, s, Xs, U, bits, group, B=B)
    torch.cuda.synchronize()
    ref = oracle_y(X, inv, c, d, z, N, bits, group, A.cpu(), B.cpu())
    assert_gemm_close(np32(Y), ref, "fused quantize + low rank", Y.dtype)
    check_quantized(ttq, W, s.cpu(), bits, group, "fused codes source")


def test_fused_quantize_projection_refusals(ttq):
    X = acts(16, 256, 113, torch.bfloat16).cuda()
    W = weights(128, 256, 114, torch.bfloat16).cuda()
    s, inv = ttq.awq_scales(ttq.act_stats(X), 16)
    Xs, _ = ttq.prepare_activations(X, inv, 4)
    with pytest.raises(ttq.TTQError):      # decode sizes: not this form
        ttq.quantize_gemm_prepared(W, s, Xs, None, 4, 64)
    X2 = acts(64, 256, 115, torch.bfloat16).cuda()
    Xs2, _ = ttq.prepare_activations(X2, inv, 4)
    with pytest.raises(ttq.TTQError):      # fp16 weights: not this form
        ttq.quantize_gemm_prepared(W.half(), s, Xs2, None, 4, 64)


# ------------------------------------- statistic fused into the epilogue ----

@pytest.mark.parametrize("T,N,K,out,pk", [
    (300, 272, 384, "bf16", 2.0),    # two token tiles, ragged N and T
    (4096, 1152, 1152, "bf16", 2.0), # many tiles, the 16-bit tensor store
    (200, 264, 256, "f32", 2.0),     # fp32 Y: the staged-tile store
    (300, 300, 256, "f16", 1.0),     # Y rows not 16-byte aligned; p = 1
    (100, 128, 256, "bf16", 3.0),
])
def test_projection_output_statistic(ttq, T, N, K, out, pk):
    """The projection's epilogue adds |Y|^p of the stored outputs per output
    channel: reduced, it equals the statistics pass over Y (the oracle's
    fp64 sums of the stored values, and the CUDA statistics kernel)."""
    X = acts(T, K, 80 + T, torch.bfloat16).cuda()
    W = weights(N, K, 81, torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s, inv = ttq.awq_scales(sums, T)
    c, d, z = ttq.quantize_rtn_grouped(W, s, 4, 64)
    Xs, _ = ttq.prepare_activations(X, inv, 4)
    if N == 300:  # a pitch whose rows are not 16-byte aligned
        big = torch.zeros((T, 301), dtype=DT[out], device="cuda")
        Y = big[:, :N]
    else:
        Y = torch.empty((T, N), dtype=DT[out], device="cuda")
    Y2, part = ttq.w_lowbit_gemm_prepared_stats(Xs, None, c, d, z, N, 4, 64,
                                                p=pk, out=Y)
    got = ttq.stats_reduce(part)
    torch.cuda.synchronize()
    Yc = np32(Y)
    ref = oracle.act_sums(Yc, pk)
    assert_rel_close(np32(got), ref, what="fused statistic")
    if N % 8 == 0:  # the statistics pass takes K % 8 == 0
        assert_rel_close(np32(got), np32(ttq.act_stats(Y.contiguous(), pk)),
                         what="fused vs statistics pass")
    # the projection itself is the plain one's
    Yp = ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, N, 4, 64,
                                    out_dtype=DT[out])
    assert torch.equal(Yp, Y.contiguous())


def test_projection_output_statistic_refusals(ttq):
    X = acts(16, 256, 90, torch.bfloat16).cuda()
    W = weights(128, 256, 91, torch.bfloat16).cuda()
    s, inv = ttq.awq_scales(ttq.act_stats(X), 16)
    c, d, z = ttq.quantize_rtn_grouped(W, s, 4, 64)
    Xs, _ = ttq.prepare_activations(X, inv, 4)
    assert ttq.projection_stats_rows(16, 128, 256, 4) == 0
    with pytest.raises(ttq.TTQError):
        ttq.w_lowbit_gemm_prepared_stats(Xs, None, c, d, z, 128, 4, 64)


# ---------------------------------------------------------- quantize ----

def dense(c, d, z, K, bits, group):
    """The GPU's padded codes/delta/zero as dense numpy arrays; checks that
    the padding is zero."""
    c = c.cpu().numpy().view(np.uint32)
    d = d.cpu().numpy()
    z = z.cpu().numpy()
    w, G = K * bits // 32, K // group
    assert not c[:, w:].any() and not d[:, G:].any() and not z[:, G:].any()
    return c[:, :w], d[:, :G], z[:, :G]


def quantize_both(ttq, W, s, bits, group):
    c, d, z = ttq.quantize_rtn_grouped(W.cuda(), None if s is None else
                                       s.cuda(), bits, group)
    s_np = None if s is None else np32(s)
    rc, rd, rz = oracle.quantize(np32(W), s_np, bits, group)
    return (*dense(c, d, z, W.shape[1], bits, group), rc, rd, rz)


def check_quantized(ttq, W, s, bits, group, what=""):
    """GPU quantizer against the oracle: bit-exact apart from counted
    near-ties. Returns the counts."""
    out = quantize_both(ttq, W, s, bits, group)
    return assert_codes_match(*out, np32(W), None if s is None else np32(s),
                              bits, group, what)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("group", [16, 32, 64, 128])
def test_quantize_bit_exact(ttq, bits, group):
    N, K = 37, 1152  # ragged rows; K not a multiple of 256
    W = weights(N, K, 100 + bits, torch.bfloat16)
    s = torch.from_numpy(np.exp(np.random.default_rng(bits).standard_normal(K)
                                * 0.7).astype(np.float32))
    check_quantized(ttq, W, s, bits, group, f"b={bits} g={group}")


def test_quantize_near_ties_are_the_only_differences(ttq):
    """Many weights at 8 bits, where near-ties are most frequent: every code
    that differs from RTN's quotient sits at a counted near-tie, and the
    zero points (an IEEE quotient on both sides) all agree."""
    W = weights(2048, 4096, 77, torch.bfloat16)
    s = torch.from_numpy(np.exp(np.random.default_rng(77).standard_normal(
        4096) * 0.7).astype(np.float32))
    for group in (16, 128):
        n_diff, weight_ties, _ = check_quantized(ttq, W, s, 8, group,
                                                 f"b=8 g={group}")
        assert weight_ties > 0 and n_diff <= weight_ties


def test_quantize_unstaged_scales_for_very_long_rows(ttq):
    """K = 28672 (a Llama-70B-sized down projection): the scales no longer
    fit the per-CTA staging buffer and are read from global memory."""
    W = weights(64, 28672, 78, torch.bfloat16)
    s = torch.from_numpy(np.exp(np.random.default_rng(78).standard_normal(
        28672) * 0.7).astype(np.float32))
    for bits, group in ((4, 128), (3, 16)):
        check_quantized(ttq, W, s, bits, group, f"K=28672 b={bits} g={group}")


@pytest.mark.parametrize("bits,seed", [(8, 40), (7, 41)])
def test_quantize_zero_point_near_ties_keep_codes_in_range(ttq, bits, seed):
    """Groups whose zero point is a near-tie (the oracle's pin search:
    rint(-mn * (1/D)) and rint(-mn / D) differ): every GPU code lies in
    [0, 2^b - 1], differs from the oracle's only at counted near-ties, and
    dequantizes within half a step of its weight."""
    from test_oracle_pins import _reciprocal_disagreements
    W, n_zero, _ = _reciprocal_disagreements(seed, bits, 12)
    assert n_zero >= 3
    Wt = torch.from_numpy(W)
    c, d, z, rc, rd, rz = quantize_both(ttq, Wt, None, bits, 16)
    assert_codes_match(c, d, z, rc, rd, rz, W, None, bits, 16, "zero ties")
    q = oracle.unpack_codes(c, 32, bits).astype(np.float64)
    assert q.max() <= (1 << bits) - 1
    dq = (q - np.repeat(z, 16, axis=1)) * np.repeat(d.astype(np.float64), 16,
                                                    axis=1)
    # half a step, plus the quotient's fp32 rounding at a near-tie (up to
    # one step of w/D, which reaches 2^b)
    bound = np.repeat(d.astype(np.float64), 16, axis=1) * (
        0.5 + 2.0 ** (bits - 22))
    assert np.all(np.abs(dq - W) <= bound)


@pytest.mark.parametrize("dt", ["f32", "f16"])
def test_quantize_dtypes_and_no_scale(ttq, dt):
    W = weights(20, 96, 9, DT[dt])
    check_quantized(ttq, W, None, 4, 32, dt)


def test_quantize_degenerate_groups(ttq):
    W = torch.zeros(4, 64)
    W[1, :16] = torch.linspace(0.1, 1.0, 16)
    W[2, 16:32] = -torch.linspace(0.1, 1.0, 16)
    W[3] = 0.5  # constant row
    c, d, z, rc, rd, rz = quantize_both(ttq, W, None, 3, 16)
    np.testing.assert_array_equal(c, rc)
    np.testing.assert_array_equal(d, rd)
    np.testing.assert_array_equal(z, rz)


def test_unpack(ttq):
    W = weights(9, 160, 3, torch.bfloat16)
    for bits in (2, 3, 5, 8):
        c, _, _ = ttq.quantize_rtn_grouped(W.cuda(), None, bits, 32)
        q = ttq.unpack_codes(c, 160, bits).cpu().numpy()
        cd = c.cpu().numpy().view(np.uint32)[:, :160 * bits // 32]
        np.testing.assert_array_equal(q, oracle.unpack_codes(cd, 160, bits))


# -------------------------------------------------------------- gemm ----

def run_path(ttq, X, W, bits, group, A=None, B=None, out_dtype=None,
             alpha=0.5, lam=0.1, p=2.0):
    """GPU path: stats -> scales -> quantize -> projection."""
    Xg, Wg = X.cuda(), W.cuda()
    sums = ttq.act_stats(Xg, p)
    s, inv = ttq.awq_scales(sums, X.shape[0], alpha, lam, p)
    c, d, z = ttq.quantize_rtn_grouped(Wg, s, bits, group)
    Y = ttq.w_lowbit_gemm(Xg, inv, c, d, z, W.shape[0], bits, group,
                          None if A is None else A.cuda(),
                          None if B is None else B.cuda(),
                          out_dtype=out_dtype)
    torch.cuda.synchronize()
    return Y, inv, c, d, z


def oracle_y(X, inv, c, d, z, N, bits, group, A=None, B=None, rows=None):
    cd, dd, zd = dense(c, d, z, X.shape[1], bits, group)
    return oracle.lowbit_gemm(np32(X), np32(inv), cd, dd, zd, N, bits, group,
                              None if A is None else np32(A),
                              None if B is None else np32(B), rows=rows)


def _prepared_order(bits):
    """Position p of a 16-channel span of the prepared operand holds channel
    order[p] of the span: the pairing of the fp16 weight pairs that b-bit
    code words unpack to (codes 8, 4 or 2 channels apart for b = 2, 4, 8),
    the layout ttq.h documents for the prepared activations."""
    p = np.arange(16)
    if bits == 2:
        return (p >> 1) + 8 * (p & 1)
    if bits == 4:
        return 8 * (p >> 3) + ((p & 7) >> 1) + 4 * (p & 1)
    if bits == 8:
        return 4 * (p >> 2) + ((p & 3) >> 1) + 2 * (p & 1)
    return p


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("T,K,pad", [(37, 288, 32), (300, 2080, 0)])
def test_prepare_activations_exact(ttq, bits, dt, T, K, pad):
    """Xs = fp16(fp32(X) * inv_s): one fp32 product rounded to fp16, bit for
    bit, in the channel order of the code width; rows of X with a pitch."""
    X = acts(T, K + pad, 80 + bits, DT[dt])
    rng = np.random.default_rng(81)
    inv = (rng.uniform(0.25, 4.0, K)).astype(np.float32)
    Xg = X.cuda()[:, :K]
    Xs, _ = ttq.prepare_activations(Xg, torch.from_numpy(inv).cuda(), bits)
    torch.cuda.synchronize()
    xf = X[:, :K].float().numpy()
    ref = (xf * inv[None, :]).astype(np.float32).astype(np.float16)
    order = _prepared_order(bits)
    idx = (np.arange(K) // 16) * 16 + order[np.arange(K) % 16]
    ref = ref[:, idx]
    got = Xs.cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("T", [1, 4, 16, 17, 100, 300])
@pytest.mark.parametrize("bits,group", [(4, 128), (3, 32), (2, 16), (5, 64)])
def test_gemm_shapes(ttq, T, bits, group):
    N, K = 300, 640  # 3 weight tiles (ragged), 10 K steps
    X = acts(T, K, 11 + T, torch.bfloat16)
    W = weights(N, K, 12, torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, bits, group)
    ref = oracle_y(X, inv, c, d, z, N, bits, group)
    assert_gemm_close(np32(Y), ref, f"T={T} b={bits} g={group}", Y.dtype)


@pytest.mark.parametrize("N,pitch", [(264, 264), (264, 320), (300, 300),
                                     (136, 136)])
@pytest.mark.parametrize("out", ["f32", "bf16", "f16"])
def test_gemm_output_tile_store(ttq, N, pitch, out):
    """Both ways the projection writes Y: 16-byte aligned rows go through
    a shared-memory tile and a tensor store (ragged N and T clipped), other
    pitches through per-row stores. Columns beyond N stay untouched."""
    T, K, bits, group = 300, 384, 4, 32
    X = acts(T, K, 31, torch.bfloat16)
    W = weights(N, K, 32, torch.bfloat16)
    Xg, Wg = X.cuda(), W.cuda()
    sums = ttq.act_stats(Xg)
    s, inv = ttq.awq_scales(sums, T)
    c, d, z = ttq.quantize_rtn_grouped(Wg, s, bits, group)
    big = torch.full((T, pitch), 7.0, dtype=DT[out], device="cuda")
    Y = big[:, :N]
    ttq.w_lowbit_gemm(Xg, inv, c, d, z, N, bits, group, out=Y)
    torch.cuda.synchronize()
    ref = oracle_y(X, inv, c, d, z, N, bits, group)
    assert_gemm_close(np32(Y), ref, f"N={N} pitch={pitch} {out}", Y.dtype)
    if pitch > N:
        assert torch.all(big[:, N:] == 7.0)


def test_one_and_two_tokens_with_very_long_rows(ttq):
    """K = 22528: one token still takes the CUDA-core product; for two
    tokens its staged activations would exceed the shared-memory budget, so
    the tensor-core decode configuration runs instead."""
    N, K = 192, 22528
    X = acts(2, K, 41, torch.bfloat16)
    W = weights(N, K, 42, torch.bfloat16)
    for T in (1, 2):
        Y, inv, c, d, z = run_path(ttq, X[:T], W, 4, 128)
        assert_gemm_close(np32(Y), oracle_y(X[:T], inv, c, d, z, N, 4, 128),
                          f"long rows T={T}", Y.dtype)


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("group", [16, 32, 128])
def test_decode_gemv(ttq, T, bits, group):
    """One or two tokens take the CUDA-core matrix-vector path, three and
    four the tensor-core decode tile; every code width and group size
    against the oracle (K spans 10 row passes of a warp's lanes and a
    ragged one)."""
    N, K = 300, 1408
    X = acts(T, K, 40 + T + bits, torch.bfloat16)
    W = weights(N, K, 41 + bits, torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, bits, group)
    ref = oracle_y(X, inv, c, d, z, N, bits, group)
    assert_gemm_close(np32(Y), ref, f"gemv T={T} b={bits} g={group}", Y.dtype)


def test_decode_gemv_many_rows_per_block(ttq):
    """160000 rows of K = 256: each CTA owns more rows than its shared
    memory holds partial sums for, so it works through them in chunks.
    Sampled output channels (first and last included) against the oracle."""
    N, K, bits, group = 160000, 256, 4, 32
    rng = np.random.default_rng(61)
    W = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(
        np.float32)).to(torch.bfloat16)
    for T in (1, 4):
        X = acts(T, K, 62 + T, torch.bfloat16)
        Y, inv, c, d, z = run_path(ttq, X, W, bits, group)
        rows = np.unique(np.concatenate([[0, N - 1], rng.choice(
            np.arange(1, N - 1), 2000, replace=False)]))
        cd, dd, zd = dense(c, d, z, K, bits, group)
        ref = oracle.lowbit_gemm(np32(X), np32(inv), cd[rows], dd[rows],
                                 zd[rows], len(rows), bits, group)
        assert_gemm_close(np32(Y)[:, rows], ref, f"many rows T={T}", Y.dtype)


@pytest.mark.parametrize("out", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("T", [1, 2, 4])
def test_decode_gemv_lowrank_and_dtypes(ttq, out, T):
    N, K, r, bits, group = 200, 512, 16, 4, 64
    X = acts(T, K, 50 + T, torch.bfloat16)
    W = weights(N, K, 51, torch.bfloat16)
    rng = np.random.default_rng(52)
    A = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32) * .05
                         ).to(torch.bfloat16)
    B = torch.from_numpy(rng.standard_normal((N, r)).astype(np.float32) * .05
                         ).to(torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, bits, group, A, B, out_dtype=DT[out])
    ref = oracle_y(X, inv, c, d, z, N, bits, group, A, B)
    assert_gemm_close(np32(Y), ref, f"gemv lowrank T={T} {out}", Y.dtype)


@pytest.mark.parametrize("bits", [6, 7, 8])
def test_gemm_wide_codes(ttq, bits):
    X = acts(64, 256, 13, torch.bfloat16)
    W = weights(160, 256, 14, torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, bits, 32)
    assert_gemm_close(np32(Y), oracle_y(X, inv, c, d, z, 160, bits, 32),
                      dtype=Y.dtype)


@pytest.mark.parametrize("K", [32, 96, 160])
def test_gemm_ragged_k(ttq, K):
    # K not a multiple of the 64-wide K step: the tail step is half empty
    X = acts(40, K, 15, torch.bfloat16)
    W = weights(130, K, 16, torch.bfloat16)
    for T in (40, 3):
        Y, inv, c, d, z = run_path(ttq, X[:T], W, 4, 32)
        assert_gemm_close(np32(Y), oracle_y(X[:T], inv, c, d, z, 130, 4, 32),
                          dtype=Y.dtype)


@pytest.mark.parametrize("T,N,K,bits,group,r,out", [
    (1542, 5770, 640, 4, 128, 0, "bf16"),   # token tile 128
    (2416, 4657, 640, 3, 32, 0, "f32"),     # token tile 160
    (2899, 4657, 640, 2, 16, 16, "f16"),    # token tile 192, low-rank stage
    (2899, 4657, 2304, 5, 128, 0, "bf16"),  # two params chunks per row tile
    (1542, 5770, 384, 8, 64, 7, "bf16"),
    (1542, 5770, 672, 3, 32, 0, "bf16"),    # ragged last K stage
    (2416, 4657, 4160, 4, 64, 16, "f32"),   # ragged K, 5 params chunks
])
def test_gemm_many_tiles_per_sm(ttq, T, N, K, bits, group, r, out):
    """Four or more output tiles per SM: each CTA walks its tiles with a
    double-buffered accumulator. Ragged N and T, into a pitched Y whose
    pad columns must stay untouched; every element written (the output is
    pre-filled with NaN), sampled token rows against the oracle."""
    X = acts(T, K, 60 + bits, torch.bfloat16)
    W = weights(N, K, 61 + bits, torch.bfloat16)
    A = B = None
    if r:
        rng = np.random.default_rng(62)
        A = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32) *
                             0.05).to(torch.bfloat16)
        B = torch.from_numpy(rng.standard_normal((N, r)).astype(np.float32) *
                             0.05).to(torch.bfloat16)
    Xg, Wg = X.cuda(), W.cuda()
    sums = ttq.act_stats(Xg)
    s, inv = ttq.awq_scales(sums, T)
    c, d, z = ttq.quantize_rtn_grouped(Wg, s, bits, group)
    pitch = N + 13
    big = torch.full((T, pitch), float("nan"), dtype=DT[out], device="cuda")
    big[:, N:] = 7.0
    Y = big[:, :N]
    ttq.w_lowbit_gemm(Xg, inv, c, d, z, N, bits, group,
                      None if A is None else A.cuda(),
                      None if B is None else B.cuda(), out=Y)
    torch.cuda.synchronize()
    assert not torch.isnan(Y).any(), "output elements left unwritten"
    assert torch.all(big[:, N:] == 7.0)
    rng = np.random.default_rng(63)
    rows = np.unique(np.concatenate([
        rng.choice(T, 40, replace=False), np.arange(T - 8, T), [0, 127, 128,
                                                               159, 160, 191,
                                                               192]]))
    ref = oracle_y(X, inv, c, d, z, N, bits, group, A, B, rows=rows)
    assert_gemm_close(np32(Y)[rows], ref, f"T={T} N={N} K={K} b={bits}",
                      Y.dtype)


@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_persistent_matches_one_tile_grid(ttq, out):
    """The persistent form (here 4096 tokens, 86 x 22 tiles) and the
    one-tile-per-CTA grid (the first 192 tokens alone: one token tile of the
    same width) run the same MMAs in the same order for a tile, so the
    first 192 rows of Y agree bit for bit. Both runs are deterministic."""
    T, N, K, bits, group = 4096, 11008, 512, 4, 128
    X = acts(T, K, 71, torch.bfloat16).cuda()
    W = weights(N, K, 72, torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s, inv = ttq.awq_scales(sums, T)
    c, d, z = ttq.quantize_rtn_grouped(W, s, bits, group)
    Y = ttq.w_lowbit_gemm(X, inv, c, d, z, N, bits, group,
                          out_dtype=DT[out])
    Y2 = ttq.w_lowbit_gemm(X, inv, c, d, z, N, bits, group,
                           out_dtype=DT[out])
    Y192 = ttq.w_lowbit_gemm(X[:192].contiguous(), inv, c, d, z, N, bits,
                             group, out_dtype=DT[out])
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    assert torch.equal(Y[:192], Y192)


@pytest.mark.parametrize("out", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("xin", ["f32", "bf16", "f16"])
def test_gemm_dtypes(ttq, xin, out):
    X = acts(50, 256, 17, DT[xin])
    W = weights(144, 256, 18, DT[xin])
    Y, inv, c, d, z = run_path(ttq, X, W, 4, 32, out_dtype=DT[out])
    assert Y.dtype == DT[out]
    assert_gemm_close(np32(Y), oracle_y(X, inv, c, d, z, 144, 4, 32),
                      dtype=Y.dtype)


def test_gemm_fp32_output_error_is_operand_rounding_only(ttq):
    # fp32 Y isolates the fp16 operand roundings (X/s and (q-z)D): far
    # below the bar
    X = acts(256, 512, 19, torch.bfloat16)
    W = weights(256, 512, 20, torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, 4, 64, out_dtype=torch.float32)
    fro, rowmax = gemm_errors(np32(Y), oracle_y(X, inv, c, d, z, 256, 4, 64))
    assert fro < 7e-4 and rowmax < 1e-2


@pytest.mark.parametrize("T", [1, 16, 200])
@pytest.mark.parametrize("r", [16, 7])
def test_gemm_lowrank(ttq, T, r):
    N, K = 272, 384
    X = acts(T, K, 21, torch.bfloat16)
    rng = np.random.default_rng(22)
    A = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32) *
                         0.05).to(torch.bfloat16)
    B = torch.from_numpy(rng.standard_normal((N, r)).astype(np.float32) *
                         0.05).to(torch.bfloat16)
    W = weights(N, K, 23, torch.bfloat16)
    Y, inv, c, d, z = run_path(ttq, X, W, 4, 64, A, B)
    assert_gemm_close(np32(Y), oracle_y(X, inv, c, d, z, N, 4, 64, A, B),
                      dtype=Y.dtype)


def test_lowrank_add_alone(ttq):
    T, K, N, r = 33, 200, 150, 16
    X = acts(T, K, 24, torch.float32)
    rng = np.random.default_rng(25)
    A = torch.from_numpy(rng.standard_normal((r, K)).astype(np.float32))
    B = torch.from_numpy(rng.standard_normal((N, r)).astype(np.float32))
    Y0 = torch.from_numpy(rng.standard_normal((T, N)).astype(np.float32))
    Y = ttq.lowrank_add(X.cuda(), A.cuda(), B.cuda(), Y0.clone().cuda())
    ref = Y0.double().numpy() + (X.double().numpy() @ A.double().numpy().T) @ \
        B.double().numpy().T
    assert_gemm_close(np32(Y), ref)


def test_gemm_deterministic_and_reusable_workspace(ttq):
    X = acts(8, 1024, 26, torch.bfloat16).cuda()
    W = weights(512, 1024, 27, torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s, inv = ttq.awq_scales(sums, 8)
    c, d, z = ttq.quantize_rtn_grouped(W, s, 4, 128)
    ws = torch.empty(ttq.workspace_size(8, 1024), dtype=torch.uint8,
                     device="cuda")
    y1 = ttq.w_lowbit_gemm(X, inv, c, d, z, 512, 4, 128, workspace=ws)
    y2 = ttq.w_lowbit_gemm(X, inv, c, d, z, 512, 4, 128, workspace=ws)
    assert torch.equal(y1, y2)


def test_fp16_range_flag(ttq):
    X = torch.full((4, 64), 60000.0, dtype=torch.float32).cuda()
    inv = torch.full((64,), 2.0, device="cuda")
    W = weights(128, 64, 28, torch.float32).cuda()
    c, d, z = ttq.quantize_rtn_grouped(W, None, 4, 32)
    ttq.device_error(clear=True)
    ttq.w_lowbit_gemm(X, inv, c, d, z, 128, 4, 32)
    assert ttq.device_error(clear=True) & ttq.DEVERR_FP16_RANGE


def test_layer_object_matches_calls(ttq):
    X = acts(64, 256, 29, torch.bfloat16).cuda()
    W = weights(96, 256, 30, torch.bfloat16).cuda()
    layer = ttq.TTQLinear(W, ttq.TTQParams(bits=3, group=32))
    y = layer(X)
    # the same calls by hand: fused statistics + scales, quantize, project
    _, s, inv = ttq.act_stats_scales(X, ttq.new_counter())
    c, d, z = ttq.quantize_rtn_grouped(W, s, 3, 32)
    Y = ttq.w_lowbit_gemm(X, inv, c, d, z, W.shape[0], 3, 32)
    assert torch.equal(y, Y)
    assert torch.equal(y, layer(X))  # the layer's counter is reusable
    # and the result agrees with the oracle
    ref = oracle_y(X.cpu(), inv, c, d, z, W.shape[0], 3, 32)
    assert_gemm_close(np32(y), ref, "layer object", y.dtype)


def test_bounded_wait_gives_up_and_leaves_the_context_usable(ttq):
    """The failure path of every in-kernel wait: a barrier that nothing
    arrives at makes the wait give up after its clock limit, raise
    TTQ_DEVERR_TIMEOUT and return; later launches still run correctly."""
    import time
    ttq.device_error(clear=True)
    done, err = ttq.selftest_bounded_wait(True)
    assert done and err == 0
    t0 = time.perf_counter()
    done, err = ttq.selftest_bounded_wait(False)
    waited = time.perf_counter() - t0
    assert not done and err & ttq.DEVERR_TIMEOUT
    assert 0.3 < waited < 30.0
    # the context is intact: a quantization after the timeout matches
    W = weights(64, 256, 5, torch.bfloat16)
    check_quantized(ttq, W, None, 4, 32, "after the timeout")
    assert ttq.device_error(clear=True) == 0
