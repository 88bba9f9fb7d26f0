"""Pins of the dynamic low-rank oracle (oracle/lowrank.py) against what the
mathematics fixes: orthonormality and triangularity of Gram-Schmidt,
numpy's Householder QR on full-rank inputs, exact recovery of low-rank
weights, the top singular subspace (numpy's SVD) and Eckart-Young's
residual at convergence, the closed form of q subspace iterations, and
hand-worked bf16 roundings.

Every pin takes the oracle module as ``lr`` so that
tests/test_lowrank_oracle_mutations.py can run the same pins against copies
with a planted mistake. TTQ review, "Proposed method", bullet 5 and "Main
results", bullet 4 (W = W_q + B A, TTQ on the residual).
"""
import numpy as np
import pytest
import torch

import oracle.lowrank as lowrank_oracle


@pytest.fixture
def lr():
    return lowrank_oracle


def _planted(N, K, k, seed, gap=0.5, noise=1e-3):
    """A matrix with k strong directions (sizes 10 gap^i) above a weak bulk,
    built from exact orthonormal factors (numpy QR of Gaussians)."""
    rng = np.random.default_rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((N, N)))
    V, _ = np.linalg.qr(rng.standard_normal((K, K)))
    m = min(N, K)
    sig = np.concatenate([10.0 * gap ** np.arange(k),
                          noise * np.linspace(1.0, 0.5, m - k)])
    return (U[:, :m] * sig[None, :]) @ V[:, :m].T


def _projector(Q):
    return Q @ Q.T


# --------------------------------------------------------- orthonormalize --

def pin_orth_full_rank(lr):
    rng = np.random.default_rng(1)
    Y = rng.standard_normal((40, 6)) * np.array([1, 5, 0.3, 2, 9, 0.7])
    Q = lr.orthonormalize(Y)
    np.testing.assert_allclose(Q.T @ Q, np.eye(6), atol=1e-12)
    R = Q.T @ Y
    np.testing.assert_allclose(np.tril(R, -1), 0.0, atol=1e-12)
    assert np.all(np.diag(R) > 0)
    np.testing.assert_allclose(Q @ R, Y, atol=1e-12)
    # numpy's Householder QR gives the same columns up to their signs
    Qh, Rh = np.linalg.qr(Y)
    np.testing.assert_allclose(Q, Qh * np.sign(np.diag(Rh))[None, :],
                               atol=1e-12)


def pin_orth_drops_dependent_and_zero_columns(lr):
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal(30), rng.standard_normal(30)
    Y = np.stack([a, 2 * a, b, np.zeros(30), a - 3 * b, a + 1e-5 * b], 1)
    Q = lr.orthonormalize(Y)
    norms = np.linalg.norm(Q, axis=0)
    np.testing.assert_allclose(norms, [1, 0, 1, 0, 0, 0], atol=1e-12)
    assert not lr.orthonormalize(np.zeros((8, 3))).any()


def pin_orth_nearly_dependent_columns_stay_orthonormal(lr):
    """Columns within a few 1e-3 of each other (condition ~1e3, above the
    drop threshold) still come out orthonormal to fp64 precision: one pass
    of Gram-Schmidt leaves errors near condition^2 x 1e-16."""
    rng = np.random.default_rng(11)
    a, b, c = rng.standard_normal((3, 200))
    Y = np.stack([a, a + 3e-3 * b, a + 3e-3 * c], 1)
    Q = lr.orthonormalize(Y)
    np.testing.assert_allclose(Q.T @ Q, np.eye(3), rtol=0, atol=1e-14)


def pin_orth_drop_threshold_is_relative(lr):
    """A column whose new part is just above tol x the largest column norm
    is kept, just below it dropped, whatever the overall scale."""
    tol = lr.DROP_TOL
    e0, e1 = np.eye(5)[:, 0], np.eye(5)[:, 1]
    for scale in (1e-6, 1.0, 1e6):
        keep = lr.orthonormalize(scale * np.stack(
            [e0, e0 + 1.01 * tol * e1], 1))
        drop = lr.orthonormalize(scale * np.stack(
            [e0, e0 + 0.99 * tol * e1], 1))
        np.testing.assert_allclose(keep[:, 1], e1, atol=1e-9)
        assert not drop[:, 1].any()
    # the reference is the largest column, wherever it stands
    e2 = np.eye(5)[:, 2]
    drop = lr.orthonormalize(np.stack([1e-2 * e2, e0, e0 + 0.99 * tol * e1],
                                      1))
    np.testing.assert_allclose(np.linalg.norm(drop, axis=0), [1, 1, 0],
                               atol=1e-12)


# ------------------------------------------------------------- factors ----

def pin_exact_low_rank_weight_is_recovered(lr):
    """A weight of rank <= r is reproduced by Q Q^T W whatever s is."""
    rng = np.random.default_rng(3)
    N, K, k, r = 48, 64, 3, 5
    W = rng.standard_normal((N, k)) @ rng.standard_normal((k, K))
    s = np.exp(rng.standard_normal(K))
    for iters in (0, 1, 2):
        Q = lr.factor_basis(W, s, rng.standard_normal((r, K)), iters)
        np.testing.assert_allclose(Q @ (Q.T @ W), W, atol=1e-9)
        assert int(np.sum(np.linalg.norm(Q, axis=0) > 0.5)) == k


def pin_converges_to_top_subspace_of_scaled_weight(lr):
    """Many iterations give the top-r left singular subspace of W diag(s)
    (numpy's SVD) and the residual energy of Eckart-Young."""
    rng = np.random.default_rng(4)
    N, K, r = 50, 70, 4
    Ws = _planted(N, K, r, 5)
    s = np.exp(0.8 * rng.standard_normal(K))
    W = Ws / s[None, :]
    Q = lr.factor_basis(W, s, rng.standard_normal((r, K)), 30)
    U, S, _ = np.linalg.svd(Ws)
    np.testing.assert_allclose(_projector(Q), _projector(U[:, :r]), atol=1e-9)
    resid = np.linalg.norm(Ws - Q @ (Q.T @ Ws)) ** 2
    np.testing.assert_allclose(resid, np.sum(S[r:] ** 2), rtol=1e-8)


def pin_subspace_is_the_scaled_weights_not_the_weights(lr):
    """W's strongest direction sits on channels with small scales: the
    factors follow W diag(s), whose strongest direction is another one."""
    rng = np.random.default_rng(9)
    N, K = 40, 60
    u1, u2 = np.linalg.qr(rng.standard_normal((N, 2)))[0].T
    v1 = np.r_[rng.standard_normal(K // 2), np.zeros(K // 2)]
    v2 = np.r_[np.zeros(K // 2), rng.standard_normal(K // 2)]
    v1, v2 = v1 / np.linalg.norm(v1), v2 / np.linalg.norm(v2)
    W = 10 * np.outer(u1, v1) + 3 * np.outer(u2, v2)
    s = np.r_[np.full(K // 2, 0.1), np.full(K // 2, 10.0)]
    Q = lr.factor_basis(W, s, rng.standard_normal((1, K)), 5)
    np.testing.assert_allclose(abs(Q[:, 0] @ u2), 1.0, atol=1e-9)


def pin_iterations_span_the_power_scheme(lr):
    """q iterations span (W_s W_s^T)^q W_s Omega^T (Halko et al., eq. of the
    power scheme), formed here without intermediate orthonormalisation."""
    rng = np.random.default_rng(6)
    N, K, r = 30, 40, 3
    W = rng.standard_normal((N, K))
    s = np.exp(0.5 * rng.standard_normal(K))
    om = rng.standard_normal((r, K))
    Ws = W * s[None, :]
    for q in (0, 1, 2):
        P = Ws @ om.T
        for _ in range(q):
            P = Ws @ (Ws.T @ P)
        Qp, _ = np.linalg.qr(P)
        Q = lr.factor_basis(W, s, om, q)
        np.testing.assert_allclose(_projector(Q), _projector(Qp), atol=1e-9)


def pin_factors_are_basis_and_projection(lr):
    """B = bf16(Q), A = bf16(Q^T W): A lives in the unscaled weight's domain
    (B A ~ W, not W diag(s))."""
    rng = np.random.default_rng(7)
    N, K, k = 24, 32, 2
    W = rng.standard_normal((N, k)) @ rng.standard_normal((k, K))
    s = np.full(K, 4.0)
    B, A = lr.dynamic_factors(W, s, rng.standard_normal((k, K)), 1)
    Q = lr.factor_basis(W, s, rng.standard_normal((k, K)), 1)
    assert np.array_equal(B, lr.round_bf16(B)) and np.array_equal(
        A, lr.round_bf16(A))
    np.testing.assert_allclose(B @ A, W, rtol=0, atol=2e-2 * np.abs(W).max())
    np.testing.assert_allclose(B.T @ B, np.eye(k), atol=1e-2)
    np.testing.assert_allclose(_projector(B), _projector(Q), atol=1e-2)


def pin_zero_weight_gives_zero_factors(lr):
    B, A = lr.dynamic_factors(np.zeros((16, 32)), np.ones(32),
                              np.ones((4, 32)), 2)
    assert not B.any() and not A.any()


# -------------------------------------------------- residual and rounding --

def pin_round_bf16_matches_torch_on_fp32_values(lr):
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(
        -30, 30, 5000), [0.0, -0.0, 1e-40, -3e-39]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    got = lr.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def pin_round_bf16_hand_worked(lr):
    # bf16 keeps 8 significant bits: at 1 the step is 2^-7; midpoints go to
    # the even neighbour, anything past a midpoint goes up
    cases = [(1 + 2.0 ** -8, 1.0), (1 + 3 * 2.0 ** -8, 1 + 2.0 ** -6),
             (1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -7),
             (-(1 + 2.0 ** -8), -1.0), (3.0, 3.0), (2.0 ** -130, 2.0 ** -130),
             (2.0 ** -134, 0.0), (3 * 2.0 ** -134, 2.0 ** -132)]
    for x, want in cases:
        assert lr.round_bf16(np.array([x]))[0] == want, x


def pin_residual_is_rounded_once(lr):
    W = np.array([[1.0, 2.0, 1.0]])
    B = np.array([[1.0]])
    A = np.array([[-2.0 ** -8, 0.5, -2.0 ** -8 - 2.0 ** -40]])
    R = lr.residual(W, B, A)
    # 1 + 2^-8 is a midpoint (to even: 1), 1.5 exact, and just above the
    # midpoint rounds up; rounding through fp32 first would lose the last one
    np.testing.assert_array_equal(R, [[1.0, 1.5, 1 + 2.0 ** -7]])
    np.testing.assert_array_equal(lr.residual(W, np.zeros((1, 2)),
                                              np.zeros((2, 3))), W)


def pin_residual_near_ties_mark_midpoints_only(lr):
    """Exact midpoints and values within the fp32 chain bound of one are
    marked; values a bf16 quarter-step away, and exact results of
    representable values, are not; a cancellation to (almost) zero is."""
    W = np.array([[1.0, 2.0, 1.0, 3.0, 1.0, 1.0]])
    B = np.array([[1.0]])
    A = np.array([[-2.0 ** -8, 0.5, -2.0 ** -8 - 2.0 ** -30,
                   -2.0 ** -9, 1.0 - 2.0 ** -40, 1.0]])
    np.testing.assert_array_equal(lr.residual_near_ties(W, B, A),
                                  [[1, 0, 1, 0, 1, 1]])


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_lowrank_oracle_pin(pin, lr):
    pin(lr)
