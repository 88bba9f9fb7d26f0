"""Parity of the per-prompt low-rank factors and the residual (the CUDA
calls ttq_lowrank_factors and ttq_lowrank_residual) with the oracle of
oracle/lowrank.py, on seeded inputs.

The factors are a basis of a subspace: what is unique is the subspace, so
the tests compare the product B A (the weight's projection onto it) and the
residual energy of the activation-scaled weight, and check that B is
orthonormal. Tolerances (derived from the arithmetic): B and A are stored in
bf16 (relative rounding 2^-9 each) and the kernels' products use fp16
operands (2^-11), so B A agrees with the oracle's to well within 1e-2
relative Frobenius when the subspace is separated from the rest of the
spectrum, and B^T B is the identity to within 1e-2. The residual energy is
stationary in the subspace (its first-order change vanishes), so it agrees
to 1e-3 relative. The residual R = bf16(W - B A) from given factors is
bit-exact except where the oracle marks a near-tie (the exact value within
the fp32 multiply-add chain's error bound of a bf16 midpoint), where it may
be one bf16 step away.

TTQ review, "Proposed method", bullet 5 and "Main results", bullet 4.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.lowrank as lr_oracle
from test_weight_quantization_b200.inputs import (activations, probe_vectors,
                                                  spectral_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ttq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_weight_quantization_b200 import ttq as mod
    return mod


def _scales(K, T, seed):
    """TTQ's scales of a seeded prompt, from the oracle (fp32)."""
    X = torch.from_numpy(activations(T, K, seed, "student_t", 0.01, 0, 30.0))
    X = X.to(torch.bfloat16).float().numpy()
    sums = oracle.act_sums(X).astype(np.float32).astype(np.float64)
    s, _ = oracle.awq_scales(sums, T, 0.5, 0.1, 2.0)
    return s.astype(np.float32)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
        torch.bfloat16)


def _run_factors(ttq, Wb, s, om, iters):
    B, A = ttq.lowrank_factors(Wb.cuda(), torch.from_numpy(s).cuda(),
                               torch.from_numpy(om).cuda(), iters)
    torch.cuda.synchronize()
    assert ttq.device_error(clear=True) == 0
    return B.double().cpu().numpy(), A.double().cpu().numpy()


def _check_factors(Bg, Ag, Bo, Ao, W, s, what, energy=True):
    P_g, P_o = Bg @ Ag, Bo @ Ao
    rel = np.linalg.norm(P_g - P_o) / max(np.linalg.norm(P_o), 1e-30)
    kept = np.linalg.norm(Bg, axis=0) > 0.5
    assert np.array_equal(kept, np.linalg.norm(Bo, axis=0) > 0.5), what
    G = Bg[:, kept].T @ Bg[:, kept]
    orth = np.abs(G - np.eye(int(kept.sum()))).max() if kept.any() else 0.0
    Eg = np.linalg.norm((W - P_g) * s[None, :]) ** 2
    Eo = np.linalg.norm((W - P_o) * s[None, :]) ** 2
    erel = abs(Eg - Eo) / max(Eo, 1e-30)
    print(f"{what}: B A rel {rel:.2e}, |B^T B - I| {orth:.2e}, "
          f"residual energy rel {erel:.2e}, kept {int(kept.sum())}")
    assert rel < 1e-2, what
    assert orth < 1e-2, what
    if energy:
        assert erel < 1e-3, what


@pytest.mark.parametrize("N,K,r,iters", [
    (640, 768, 16, 1),     # several tiles, whole stages
    (300, 520, 7, 2),      # ragged rows, ragged contraction, odd rank
    (1152, 1152, 16, 0),   # the range finder alone
    (200, 1032, 32, 1),    # two 16-wide MMA column blocks
    (384, 256, 64, 1),     # the largest rank
])
def test_factors_match_oracle(ttq, N, K, r, iters):
    W = spectral_weights(N, K, 100 + N, strong=r, sigma0=20.0, decay=0.9)
    Wb = _bf16(W)
    Wd = Wb.double().numpy()
    s = _scales(K, 256, 200 + K)
    om = probe_vectors(r, K, 300 + r)
    Bg, Ag = _run_factors(ttq, Wb, s, om, iters)
    Bo, Ao = lr_oracle.dynamic_factors(Wd, s, om, iters)
    _check_factors(Bg, Ag, Bo, Ao, Wd, s.astype(np.float64),
                   f"{N}x{K} r={r} iters={iters}")


def test_factors_of_exactly_low_rank_weight_drop_columns(ttq):
    """A bf16-exact weight of rank 3 with r = 8: three kept columns, five
    zero ones, and B A = W up to the bf16 rounding of B and A."""
    rng = np.random.default_rng(5)
    N, K, r = 260, 384, 8
    # every sum of three such products has at most 7 significant bits
    vals = np.array([-2.0, -1.0, 1.0, 2.0])
    U = rng.choice(vals, size=(N, 3))
    V = rng.choice(vals, size=(3, K)) * np.array([[1.0], [2.0 ** -3],
                                                  [2.0 ** -4]])
    W = U @ V
    Wb = _bf16(W)
    assert np.array_equal(Wb.double().numpy(), W)
    s = _scales(K, 128, 11)
    om = probe_vectors(r, K, 12)
    Bg, Ag = _run_factors(ttq, Wb, s, om, 1)
    kept = np.linalg.norm(Bg, axis=0) > 0.5
    assert kept.sum() == 3 and not Bg[:, ~kept].any() and not Ag[~kept].any()
    np.testing.assert_allclose(Bg @ Ag, W, rtol=0, atol=2e-2 * np.abs(W).max())
    Bo, Ao = lr_oracle.dynamic_factors(W, s, om, 1)
    # the residual of an exactly low-rank weight is the rounding of B and A
    # alone, different on the two sides: its energy is not compared
    _check_factors(Bg, Ag, Bo, Ao, W, s.astype(np.float64), "rank 3",
                   energy=False)


def test_factors_with_rank_above_the_dimension(ttq):
    """r = 48 > N = 40: the basis spans all 40 rows (B A = W) and the last
    eight columns are dropped."""
    N, K, r = 40, 256, 48
    W = spectral_weights(N, K, 21, strong=8)
    Wb = _bf16(W)
    s = _scales(K, 64, 22)
    om = probe_vectors(r, K, 23)
    Bg, Ag = _run_factors(ttq, Wb, s, om, 1)
    kept = np.linalg.norm(Bg, axis=0) > 0.5
    assert kept.sum() == N and not kept[N:].any()
    Wd = Wb.double().numpy()
    rel = np.linalg.norm(Bg @ Ag - Wd) / np.linalg.norm(Wd)
    assert rel < 1e-2, rel


def test_factors_of_zero_weight_are_zero(ttq):
    N, K, r = 130, 136, 16
    Wb = torch.zeros(N, K, dtype=torch.bfloat16)
    s = np.ones(K, np.float32)
    Bg, Ag = _run_factors(ttq, Wb, s, probe_vectors(r, K, 1), 2)
    assert not Bg.any() and not Ag.any()


def test_factors_are_deterministic_and_reuse_the_workspace(ttq):
    N, K, r = 512, 640, 16
    Wb = _bf16(spectral_weights(N, K, 31, strong=r)).cuda()
    s = torch.from_numpy(_scales(K, 128, 32)).cuda()
    om = torch.from_numpy(probe_vectors(r, K, 33)).cuda()
    ws = torch.empty(ttq.lowrank_factors_workspace_size(N, K, r),
                     dtype=torch.uint8, device="cuda")
    outs = [ttq.lowrank_factors(Wb, s, om, 1, workspace=ws) for _ in range(3)]
    torch.cuda.synchronize()
    assert ttq.device_error(clear=True) == 0
    for B, A in outs[1:]:
        assert torch.equal(B, outs[0][0]) and torch.equal(A, outs[0][1])


@pytest.mark.parametrize("N,K,r", [(300, 520, 7), (512, 4096, 16),
                                   (64, 1000, 32), (33, 264, 64)])
def test_residual_matches_oracle(ttq, N, K, r):
    W = spectral_weights(N, K, 40 + r, strong=r)
    Wb = _bf16(W)
    Wd = Wb.double().numpy()
    s = _scales(K, 128, 41)
    Bo, Ao = lr_oracle.dynamic_factors(Wd, s, probe_vectors(r, K, 42), 1)
    Ro = lr_oracle.residual(Wd, Bo, Ao)
    tie = lr_oracle.residual_near_ties(Wd, Bo, Ao)
    Rg = ttq.lowrank_residual(Wb.cuda(), _bf16(Bo).cuda(), _bf16(Ao).cuda())
    torch.cuda.synchronize()
    Rg = Rg.double().cpu().numpy()
    diff = Rg != Ro
    print(f"residual {N}x{K} r={r}: {int(diff.sum())} differ, "
          f"{int(tie.sum())} near-ties of {Rg.size}")
    assert not (diff & ~tie).any()
    # where they differ, by one bf16 step
    step = np.ldexp(1.0, np.frexp(np.maximum(np.abs(Ro), 1e-38))[1] - 8)
    assert np.all(np.abs(Rg - Ro)[diff] <= step[diff] * 1.0001)


def test_residual_in_place_and_pitched(ttq):
    N, K, r = 96, 520, 16
    W = spectral_weights(N, K, 50, strong=r)
    Wd = _bf16(W).double().numpy()
    s = _scales(K, 64, 51)
    Bo, Ao = lr_oracle.dynamic_factors(Wd, s, probe_vectors(r, K, 52), 1)
    ref = ttq.lowrank_residual(_bf16(Wd).cuda(), _bf16(Bo).cuda(),
                               _bf16(Ao).cuda())
    big = torch.zeros(N, K + 24, dtype=torch.bfloat16, device="cuda")
    big[:, :K] = _bf16(Wd).cuda()
    Wv = big[:, :K]
    out = ttq.lowrank_residual(Wv, _bf16(Bo).cuda(), _bf16(Ao).cuda(), out=Wv)
    torch.cuda.synchronize()
    assert out.data_ptr() == Wv.data_ptr()
    assert torch.equal(Wv, ref) and not big[:, K:].any()


def test_dynamic_low_rank_layer_beats_plain_ttq(ttq):
    """The whole per-prompt path on the GPU (statistics, scales, factors,
    residual, quantization of the residual, projection with the low-rank
    term) against the oracle's own run of the same path: on a weight with
    a strong low-rank part the output error against the exact projection
    is that of the oracle's path (within 10 %), and well below plain
    TTQ's."""
    N, K, T, r, bits, group = 512, 768, 256, 16, 4, 64
    W = _bf16(spectral_weights(N, K, 60, strong=r))
    X = _bf16(activations(T, K, 61, "gauss", 0.01, 0, 20.0))
    om = probe_vectors(r, K, 62)
    Xc, Wc = X.cuda(), W.cuda()
    sums = ttq.act_stats(Xc)
    s, inv = ttq.awq_scales(sums, T)
    B, A = ttq.lowrank_factors(Wc, s, torch.from_numpy(om).cuda(), 1)
    R = ttq.lowrank_residual(Wc, B, A)
    c, d, z = ttq.quantize_rtn_grouped(R, s, bits, group)
    Y = ttq.w_lowbit_gemm(Xc, inv, c, d, z, N, bits, group, A, B,
                          out_dtype=torch.float32)
    c2, d2, z2 = ttq.quantize_rtn_grouped(Wc, s, bits, group)
    Yp = ttq.w_lowbit_gemm(Xc, inv, c2, d2, z2, N, bits, group,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert ttq.device_error(clear=True) == 0
    Xd, Wd = X.double().numpy(), W.double().numpy()
    ref = Xd @ Wd.T
    so = oracle.act_sums(Xd.astype(np.float32)).astype(np.float32)
    s_o, inv_o = oracle.awq_scales(so.astype(np.float64), T, 0.5, 0.1, 2.0)
    s_o, inv_o = s_o.astype(np.float32), inv_o.astype(np.float32)
    Bo, Ao = lr_oracle.dynamic_factors(Wd, s_o, om, 1)
    Ro = lr_oracle.residual(Wd, Bo, Ao)
    co, do, zo = oracle.quantize(Ro.astype(np.float32), s_o, bits, group)
    Yo = oracle.lowbit_gemm(Xd.astype(np.float32), inv_o, co, do, zo, N, bits,
                            group, Ao.astype(np.float32),
                            Bo.astype(np.float32))

    def err(Yv):
        return np.linalg.norm(Yv - ref) / np.linalg.norm(ref)

    e_gpu, e_o = err(Y.double().cpu().numpy()), err(Yo)
    e_plain = err(Yp.double().cpu().numpy())
    print(f"dynamic low rank: gpu {e_gpu:.4f}, oracle {e_o:.4f}, "
          f"plain TTQ {e_plain:.4f}")
    assert e_gpu < 1.1 * e_o
    assert e_gpu < 0.5 * e_plain


def test_factors_at_llama_size(ttq):
    """A 4096 x 4096 layer (Llama-7B attention) at rank 16 with one
    iteration, against the oracle at full size."""
    N = K = 4096
    r = 16
    W = spectral_weights(N, K, 70, strong=r)
    Wb = _bf16(W)
    Wd = Wb.double().numpy()
    s = _scales(K, 256, 71)
    om = probe_vectors(r, K, 72)
    Bg, Ag = _run_factors(ttq, Wb, s, om, 1)
    Bo, Ao = lr_oracle.dynamic_factors(Wd, s, om, 1)
    _check_factors(Bg, Ag, Bo, Ao, Wd, s.astype(np.float64), "4096x4096")
