"""Oracle of the per-prompt ("dynamic") low-rank factors, fp64 numpy.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product package never imports it,
and it imports nothing of the product package.

TTQ review, "Proposed method", bullet 5: when needed, W is written as
W_q + B A with dynamic low-rank factors B and A, and W_q is quantized on the
fly; "Main results", bullet 4: TTQ then quantizes the residual and adds the
low-rank projection. The pages do not say how B and A are found. The
reading taken here: per prompt, after TTQ's scales s are known, the factors
span the dominant r-dimensional column space of the activation-scaled weight
W diag(s) (the matrix TTQ quantizes), found by randomized subspace
iteration (Halko, Martinsson and Tropp, "Finding structure with
randomness", SIAM Review 2011, Algorithm 4.4) from r Gaussian probe vectors
that the caller draws:

    Q = orth(W_s Omega^T)
    repeat ``iters`` times:  Z = orth(W_s^T Q);  Q = orth(W_s Z)
    B = Q,  A = Q^T W          (so B A = Q Q^T W, the weight's projection)

with W_s = W diag(s) and Omega [r, K] the probe vectors. B and A are stored
in bf16, the factor format of the projection; the residual W - B A is
formed from the stored factors and rounded to bf16 once.

``orth`` is Gram-Schmidt against the columns kept so far, applied twice,
with one rule of its own: a column whose part orthogonal to the kept columns
has a norm of at most ``DROP_TOL`` times the largest column norm of its
input is dropped (its output column is zero). Exactly rank-deficient
inputs (a zero weight, a weight of rank below r) then give zero columns
instead of arbitrary directions.
"""
from __future__ import annotations

import numpy as np

DROP_TOL = 2.0 ** -10


def orthonormalize(Y, tol: float = DROP_TOL) -> np.ndarray:
    """Orthonormal columns Q [M, l] spanning the columns of Y [M, l] in
    order (Q^T Y upper triangular with a non-negative diagonal); columns
    weaker than ``tol`` times the largest input column are dropped (zero)."""
    Y = np.asarray(Y, dtype=np.float64)
    M, l = Y.shape
    Q = np.zeros((M, l), np.float64)
    ref = float(np.max(np.linalg.norm(Y, axis=0))) if l else 0.0
    kept: list[int] = []
    for j in range(l):
        v = Y[:, j].copy()
        for _ in range(2):
            for i in kept:
                v -= (Q[:, i] @ v) * Q[:, i]
        nv = float(np.linalg.norm(v))
        if ref > 0.0 and nv > tol * ref:
            Q[:, j] = v / nv
            kept.append(j)
    return Q


def factor_basis(W, s, omega, iters: int) -> np.ndarray:
    """Q [N, r] fp64: the orthonormal basis of randomized subspace
    iteration on W diag(s) from the probe vectors omega [r, K]."""
    W = np.asarray(W, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    omega = np.asarray(omega, dtype=np.float64)
    Ws = W * s[None, :]
    Q = orthonormalize(Ws @ omega.T)
    for _ in range(int(iters)):
        Z = orthonormalize(Ws.T @ Q)
        Q = orthonormalize(Ws @ Z)
    return Q


def round_bf16(x) -> np.ndarray:
    """Round-to-nearest-even of fp64 values to bf16 (8 significant bits,
    the exponent range of fp32), returned as fp64; one rounding."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # below 2^-126: the subnormal step
    step_exp = e - 8                        # 8 significant bits
    return np.ldexp(np.rint(np.ldexp(x, -step_exp)), step_exp)


def dynamic_factors(W, s, omega, iters: int):
    """(B [N, r], A [r, K]) as bf16 values in fp64 arrays: B = Q and
    A = Q^T W, each rounded to bf16 once."""
    W = np.asarray(W, dtype=np.float64)
    Q = factor_basis(W, s, omega, iters)
    return round_bf16(Q), round_bf16(Q.T @ W)


def residual(W, B, A) -> np.ndarray:
    """R = W - B A from the stored factors, rounded to bf16 once."""
    W = np.asarray(W, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    return round_bf16(W - B @ A)


def residual_near_ties(W, B, A) -> np.ndarray:
    """Where a residual computed in fp32 may round to the other bf16
    neighbour: the exact W - B A lies within the bound of an fp32
    multiply-add chain over r terms, (r + 1) 2^-24 (|W| + sum_j |B_j A_j|),
    of a point halfway between two bf16 values. Elsewhere every such
    computation gives the bf16 value of ``residual``."""
    W = np.asarray(W, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    r = B.shape[1]
    v = W - B @ A
    bound = (r + 1) * 2.0 ** -24 * (np.abs(W) + np.abs(B) @ np.abs(A))
    m, e = np.frexp(v)
    e = np.maximum(e, -125)
    step = np.ldexp(1.0, e - 8)
    # distance to the nearest midpoint between bf16 neighbours
    frac = v / step - np.floor(v / step)
    dist = np.abs(frac - 0.5) * step
    # (a value within the bound of zero may round to any of the tiny bf16
    # values around it)
    return (dist <= bound) | (np.abs(v) <= bound)
