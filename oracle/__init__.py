"""Python front of the plain-C TTQ oracle (``ttq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product package never imports it.
It does not import the product package either.

Every function takes and returns numpy arrays on the host. Floating inputs
are passed to C as float32 (bf16 and fp16 values convert exactly); statistics,
scales, GEMM and loss come back in float64, the quantizer's outputs in the
storage types of the format (uint32 codes, float32 delta, uint8 zero).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ttq_oracle.c")
# TTQ_ORACLE_LIB names a prebuilt variant of this library instead (the tests
# that plant a mistake in a copy of the source and check that a pin fails).
_VARIANT = os.environ.get("TTQ_ORACLE_LIB")
_LIB = _VARIANT or os.path.join(_HERE, "libttq_oracle.so")

# -ffp-contract=off and no -ffast-math: the quantizer's fp32 arithmetic must be
# exactly the IEEE operations written in the source.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fexcess-precision=standard"]


def build(force: bool = False) -> str:
    """Compiles the oracle with gcc if the library is missing or stale."""
    if _VARIANT:
        return _LIB
    if (force or not os.path.exists(_LIB)
            or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        D = ctypes.c_double
        lib.oracle_act_sums.argtypes = [P, I64, I64, I64, D, P]
        lib.oracle_awq_scales.argtypes = [P, I64, I64, D, D, D, P, P]
        lib.oracle_awq_scales_given_mean.argtypes = [P, I64, I64, D, D, D, D,
                                                     P, P]
        lib.oracle_pack_codes.argtypes = [P, I64, I64, I, P]
        lib.oracle_unpack_codes.argtypes = [P, I64, I64, I, P]
        lib.oracle_quantize.argtypes = [P, I64, I64, I64, P, I, I, P, P, P]
        lib.oracle_count_near_ties.argtypes = [P, I64, I64, I64, P, I, I]
        lib.oracle_count_near_ties.restype = I64
        lib.oracle_near_tie_mask.argtypes = [P, I64, I64, I64, P, I, I, P, P]
        lib.oracle_near_tie_mask.restype = I64
        lib.oracle_dequantize.argtypes = [P, P, P, I64, I64, I, I, P]
        lib.oracle_lowbit_gemm.argtypes = [P, I64, I64, I64, P, I64, P, P, P,
                                           P, I64, I, I, P, P, I, P]
        lib.oracle_loss.argtypes = [P, I64, I64, P, P, I64]
        lib.oracle_loss.restype = D
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def act_sums(X, p: float = 2.0) -> np.ndarray:
    """sum_t |X[t, j]|^p per channel j, fp64 (step 1)."""
    X = _f32(X)
    T, K = X.shape
    out = np.zeros(K, np.float64)
    _load().oracle_act_sums(_ptr(X), T, K, K, float(p), _ptr(out))
    return out


def awq_scales(sums, T_total: int, alpha: float, lam: float, p: float):
    """(s, inv_s) in fp64 from per-channel sums (step 2)."""
    sums = np.ascontiguousarray(np.asarray(sums, dtype=np.float64))
    K = sums.shape[0]
    s = np.empty(K, np.float64)
    inv = np.empty(K, np.float64)
    _load().oracle_awq_scales(_ptr(sums), int(T_total), K, float(alpha),
                              float(lam), float(p), _ptr(s), _ptr(inv))
    return s, inv


def awq_scales_given_mean(sums, T_total: int, mbar: float, alpha: float,
                          lam: float, p: float):
    """(s, inv_s) in fp64 of a shard of channels whose shrinkage mean mbar
    is taken over all channels (step 2)."""
    sums = np.ascontiguousarray(np.asarray(sums, dtype=np.float64))
    K = sums.shape[0]
    s = np.empty(K, np.float64)
    inv = np.empty(K, np.float64)
    _load().oracle_awq_scales_given_mean(_ptr(sums), int(T_total), K,
                                         float(mbar), float(alpha), float(lam),
                                         float(p), _ptr(s), _ptr(inv))
    return s, inv


def quantize(W, s, bits: int, group: int):
    """Group RTN of W * diag(s) in fp32 (step 3).

    Returns (codes uint32 [N, K*bits/32], delta float32 [N, K/g],
    zero uint8 [N, K/g]). ``s`` may be None (all ones); it is rounded to
    float32 before use, as the format stores it.
    """
    W = _f32(W)
    N, K = W.shape
    s32 = None if s is None else _f32(s)
    codes = np.zeros((N, K * bits // 32), np.uint32)
    delta = np.zeros((N, K // group), np.float32)
    zero = np.zeros((N, K // group), np.uint8)
    _load().oracle_quantize(_ptr(W), N, K, K, _ptr(s32), bits, group,
                            _ptr(codes), _ptr(delta), _ptr(zero))
    return codes, delta, zero


def count_near_ties(W, s, bits: int, group: int) -> int:
    """Weights whose pre-round quotient w/D is within one fp32 step of a
    half-integer (see near_tie_mask)."""
    W = _f32(W)
    N, K = W.shape
    s32 = None if s is None else _f32(s)
    return int(_load().oracle_count_near_ties(_ptr(W), N, K, K, _ptr(s32),
                                              bits, group))


def near_tie_mask(W, s, bits: int, group: int):
    """Where two valid fp32 evaluations of the quantizer may disagree.

    Returns (mask uint8 [N, K], weight_ties, group_ties): bit 0 of mask is
    set where the weight's own quotient w/D lies within one fp32 step of a
    half-integer, bit 1 where its group's zero-point quotient -mn/D does (any
    code of the group may move with it); the counts are of such weights and
    of such groups.
    """
    W = _f32(W)
    N, K = W.shape
    s32 = None if s is None else _f32(s)
    mask = np.zeros((N, K), np.uint8)
    groups = ctypes.c_int64(0)
    weights = _load().oracle_near_tie_mask(_ptr(W), N, K, K, _ptr(s32), bits,
                                           group, _ptr(mask),
                                           ctypes.byref(groups))
    return mask, int(weights), int(groups.value)


def pack_codes(q, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(np.asarray(q, dtype=np.uint8))
    N, K = q.shape
    codes = np.zeros((N, K * bits // 32), np.uint32)
    _load().oracle_pack_codes(_ptr(q), N, K, bits, _ptr(codes))
    return codes


def unpack_codes(codes, K: int, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint32))
    N = codes.shape[0]
    q = np.zeros((N, K), np.uint8)
    _load().oracle_unpack_codes(_ptr(codes), N, K, bits, _ptr(q))
    return q


def dequantize(codes, delta, zero, K: int, bits: int, group: int):
    """Scaled-domain weight (q - z) * delta in fp64, [N, K]."""
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint32))
    delta = _f32(delta)
    zero = np.ascontiguousarray(np.asarray(zero, dtype=np.uint8))
    N = codes.shape[0]
    out = np.zeros((N, K), np.float64)
    _load().oracle_dequantize(_ptr(codes), _ptr(delta), _ptr(zero), N, K,
                              bits, group, _ptr(out))
    return out


def lowbit_gemm(X, inv_s, codes, delta, zero, N: int, bits: int, group: int,
                A=None, B=None, rows=None) -> np.ndarray:
    """Y = (X diag(inv_s)) W_hat_s^T [+ (X A^T) B^T] in fp64 (step 4).

    ``rows`` selects token rows (the result has one row per entry).
    """
    X = _f32(X)
    T, K = X.shape
    inv_s = _f32(inv_s)
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint32))
    delta = _f32(delta)
    zero = np.ascontiguousarray(np.asarray(zero, dtype=np.uint8))
    r = 0
    if A is not None:
        A = _f32(A)
        B = _f32(B)
        r = A.shape[0]
    rows_arr = None
    n_rows = T
    if rows is not None:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows = rows_arr.shape[0]
    Y = np.zeros((n_rows, N), np.float64)
    _load().oracle_lowbit_gemm(_ptr(X), T, K, K, _ptr(rows_arr), n_rows,
                               _ptr(inv_s), _ptr(codes), _ptr(delta),
                               _ptr(zero), N, bits, group, _ptr(A), _ptr(B),
                               r, _ptr(Y))
    return Y


def loss(W, W_eff, X) -> float:
    """L = (1/T) ||(W - W_eff) X^T||_F^2 in fp64 (the objective)."""
    W = _f32(W)
    W_eff = np.ascontiguousarray(np.asarray(W_eff, dtype=np.float64))
    X = _f32(X)
    N, K = W.shape
    T = X.shape[0]
    return float(_load().oracle_loss(_ptr(W), N, K, _ptr(W_eff), _ptr(X), T))


def effective_weight(codes, delta, zero, s, K: int, bits: int, group: int):
    """W_eff[n, j] = (q - z) * delta / s_j in fp64."""
    What = dequantize(codes, delta, zero, K, bits, group)
    if s is None:
        return What
    return What / np.asarray(s, dtype=np.float32).astype(np.float64)[None, :]
