"""The projection entry point that needs no caller workspace.

ttq_w_lowbit_gemm_noalloc serves callers that cannot allocate device memory
where they run the projection (an engine plugin called after the engine fixed
its memory plan, or host code that only holds device pointers handed to it):
its scratch is an array built into the library. These tests call it through
the C ABI and check that, on two calls in a row, it returns what the
workspace entry point ttq_w_lowbit_gemm returns (within the projection
tolerance of the parity tests, and bit for bit, since both run the same
deterministic kernels), and that inputs too large for the built-in scratch
are refused without a launch.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity_util import assert_gemm_close, np32

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20  # TTQ_NOALLOC_SCRATCH_BYTES in ttq.h


@pytest.fixture(scope="module")
def ttq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from test_weight_quantization_b200 import ttq as mod
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fn = mod._lib.ttq_w_lowbit_gemm_noalloc
    fn.argtypes = [P, I, I64, I64, I64, P, P, P, P, I64, I, I, P, P, I, P, I,
                   I64, P]
    fn.restype = I
    return mod


def noalloc(ttq, X, inv, c, d, z, N, bits, group, Y, A=None, B=None):
    dt = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}
    T, K = X.shape
    r = 0 if A is None else A.shape[0]
    return ttq._lib.ttq_w_lowbit_gemm_noalloc(
        X.data_ptr(), dt[X.dtype], T, K, X.stride(0), inv.data_ptr(),
        c.data_ptr(), d.data_ptr(), z.data_ptr(), N, bits, group,
        None if A is None else A.data_ptr(), None if B is None else B.data_ptr(),
        r, Y.data_ptr(), dt[Y.dtype], Y.stride(0),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,N,K,bits,group,r", [
    (64, 640, 768, 4, 32, 0),     # prefill tile shape, several K stages
    (4, 300, 512, 3, 16, 0),      # decode configuration, ragged rows
    (200, 272, 384, 4, 64, 16),   # with the low-rank stage
    (1, 300, 512, 4, 32, 0),      # one token: the CUDA-core product
    (2, 272, 384, 3, 32, 16),     # two tokens with the low-rank term
])
def test_noalloc_matches_workspace_entry_point(ttq, T, N, K, bits, group, r):
    g = torch.Generator().manual_seed(T + N + K)
    X = torch.randn(T, K, generator=g).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    A = B = None
    if r:
        A = (torch.randn(r, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
        B = (torch.randn(N, r, generator=g) * 0.05).to(torch.bfloat16).cuda()
    sums = ttq.act_stats(X)
    s, inv = ttq.awq_scales(sums, T)
    c, d, z = ttq.quantize_rtn_grouped(W, s, bits, group)
    ref = ttq.w_lowbit_gemm(X, inv, c, d, z, N, bits, group, A, B)
    outs = []
    for _ in range(2):  # the shared scratch keeps the previous call's data
        Y = torch.full((T, N), float("nan"), dtype=torch.bfloat16,
                       device="cuda")
        assert noalloc(ttq, X, inv, c, d, z, N, bits, group, Y, A, B) == 0
        outs.append(Y)
    torch.cuda.synchronize()
    assert ttq.device_error(clear=True) == 0
    for Y in outs:
        assert_gemm_close(np32(Y), np32(ref).astype(np.float64),
                          "noalloc vs workspace", Y.dtype)
        assert torch.equal(Y, ref)


def test_noalloc_refuses_inputs_beyond_its_scratch(ttq):
    """The limit is exact: 2048 tokens of 4096 channels fill the scratch
    (2048 * 4096 * 2 bytes) and run; one token more, or the same tokens with
    a low-rank term, is refused with nothing launched."""
    K, N = 4096, 128
    assert ttq.workspace_size(2048, K) == SCRATCH_BYTES
    assert ttq.workspace_size(2049, K) > SCRATCH_BYTES
    assert ttq.workspace_size(2048, K, 16) > SCRATCH_BYTES
    X = torch.zeros(2049, K, dtype=torch.bfloat16, device="cuda")
    inv = torch.ones(K, device="cuda")
    c = torch.zeros(N, ttq.codes_ld(K, 4), dtype=torch.int32, device="cuda")
    d = torch.zeros(N, ttq.groups_ld(K, 128), device="cuda")
    z = torch.zeros(N, ttq.groups_ld(K, 128), dtype=torch.uint8, device="cuda")
    A = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(N, 16, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((2049, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert noalloc(ttq, X, inv, c, d, z, N, 4, 128, Y) == 2  # UNSUPPORTED
    assert noalloc(ttq, X[:2048], inv, c, d, z, N, 4, 128, Y[:2048], A,
                   B) == 2
    torch.cuda.synchronize()
    assert torch.all(Y == 7.0)
    # the exact fit runs (zero weights give a zero projection)
    assert noalloc(ttq, X[:2048], inv, c, d, z, N, 4, 128, Y[:2048]) == 0
    torch.cuda.synchronize()
    assert ttq.device_error(clear=True) == 0
    assert not Y[:2048].any() and torch.all(Y[2048:] == 7.0)
