"""Shared helpers of the GPU parity tests (comparison rules only; no method
arithmetic). Tolerances are the ones the parity contract fixes:
statistics and scales 1e-5 relative; GEMM relative Frobenius error 2e-3 and
max-abs error at most 1e-2 of the reference row's RMS; step sizes bit-exact;
codes and zero points bit-exact except at the near-ties the oracle marks
(a quotient within one fp32 step of a half-integer), which are counted.

A projection stored in bf16 or fp16 cannot be closer to the exact value than
half an ulp of that type; the max-abs bar therefore applies to the error in
excess of that final rounding (for fp32 outputs the allowance is zero). The
Frobenius bar includes the final rounding."""
import numpy as np
import torch

import oracle

STATS_RTOL = 1e-5
GEMM_FRO = 2e-3
GEMM_ROWMAX = 1e-2


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def assert_rel_close(got, ref, rtol=STATS_RTOL, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    denom = np.maximum(np.abs(ref), 1e-30)
    err = np.abs(got - ref) / denom
    bad = err > rtol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} exceed "
                           f"{rtol}; worst {err.max():.3e}")


MANTISSA_BITS = {torch.bfloat16: 7, torch.float16: 10, torch.float32: None}


def half_ulp(ref, dtype):
    """Half an ulp of ``dtype`` at each |ref| (0 for fp32 outputs)."""
    m = MANTISSA_BITS.get(dtype)
    if m is None:
        return np.zeros_like(ref)
    a = np.maximum(np.abs(ref), 1e-30)
    e = np.floor(np.log2(a))
    if dtype == torch.float16:
        e = np.maximum(e, -14.0)  # subnormal spacing
    return np.ldexp(1.0, (e - m - 1).astype(np.int64))


def gemm_errors(Y, ref, dtype=torch.float32):
    Y = np.asarray(Y, np.float64)
    ref = np.asarray(ref, np.float64)
    fro = np.linalg.norm(Y - ref) / max(np.linalg.norm(ref), 1e-300)
    rms = np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True))
    excess = np.maximum(np.abs(Y - ref) - half_ulp(ref, dtype), 0.0)
    rowmax = np.max(excess / np.maximum(rms, 1e-300))
    return fro, rowmax


def assert_gemm_close(Y, ref, what="", dtype=torch.float32):
    fro, rowmax = gemm_errors(Y, ref, dtype)
    assert fro <= GEMM_FRO, f"{what}: relative Frobenius error {fro:.3e}"
    assert rowmax <= GEMM_ROWMAX, f"{what}: max |err| / row RMS {rowmax:.3e}"
    return fro, rowmax


def assert_codes_match(gc, gd, gz, rc, rd, rz, W, s, bits, group, what=""):
    """GPU codes/delta/zero (dense numpy) against the oracle's for the
    weights W (fp32 numpy, the rows both quantized) and scales s.

    delta must be bit-exact. A zero point may differ only in a group whose
    zero-point quotient is a near-tie; a code only where its own quotient or
    its group's zero-point quotient is one. Returns (codes that differ,
    weight near-ties, zero-point near-tie groups) and prints them."""
    N, K = W.shape
    np.testing.assert_array_equal(gd, rd, err_msg=f"{what} delta")
    mask, weight_ties, group_ties = oracle.near_tie_mask(W, s, bits, group)
    zero_tie = (mask[:, ::group] & 2) != 0
    zbad = (gz != rz) & ~zero_tie
    assert not zbad.any(), f"{what}: {int(zbad.sum())} zero points differ"
    diff = oracle.unpack_codes(gc, K, bits) != oracle.unpack_codes(rc, K,
                                                                   bits)
    bad = diff & (mask == 0)
    assert not bad.any(), (f"{what}: {int(bad.sum())} codes differ away "
                           f"from a near-tie (first at "
                           f"{tuple(np.argwhere(bad)[0])})")
    n_diff = int(diff.sum())
    print(f"{what}: {n_diff} of {diff.size} codes differ, all at near-ties "
          f"({weight_ties} weight near-ties, {group_ties} zero-point "
          f"near-tie groups)")
    return n_diff, weight_ties, group_ties
