"""ctypes binding of libttq (include/ttq.h): same call names, marshalling only.

Every function takes torch tensors that already live on a CUDA device,
passes their device pointers and the current torch stream to the C ABI, and
raises :class:`TTQError` on a non-OK status. No step of the computation runs
in Python; if ``libttq.so`` is missing or cannot be loaded, importing this
module raises, so there is no silent fallback.

Paper: "TTQ: Activation-Aware Test-Time Quantization to Accelerate LLM
Inference On The Fly" (TTQ review, section "Proposed method", bullets 1-7).
"""
from __future__ import annotations

import ctypes
import functools
import os
from dataclasses import dataclass

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libttq.so")

TTQ_OK = 0
DEVERR_TIMEOUT = 0x1
DEVERR_FP16_RANGE = 0x2

_DTYPE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


class TTQError(RuntimeError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build it with "
            "`python -m test_weight_quantization_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I, F, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                        ctypes.c_float, ctypes.c_size_t)
    sig = {
        "ttq_act_stats": [P, I, I64, I64, I64, F, I, P, P],
        "ttq_awq_scales": [P, I64, I64, P, P, P, P],
        "ttq_act_stats_scales": [P, I, I64, I64, I64, I, I64, P, P, P, P, P,
                                 P],
        "ttq_quantize_rtn_grouped": [P, I, I64, I64, I64, P, I, I, P, P, P, P],
        "ttq_w_lowbit_gemm_workspace_size": [I64, I64, I],
        "ttq_w_lowbit_gemm": [P, I, I64, I64, I64, P, P, P, P, I64, I, I, P, P,
                              I, P, I, I64, P, SZ, P],
        "ttq_prepare_activations": [P, I, I64, I64, I64, P, I, P, I, P, P, P],
        "ttq_w_lowbit_gemm_prepared": [P, P, I64, I64, P, P, P, I64, I, I, P,
                                       I, I, P, I, I64, P],
        "ttq_lowrank_add": [P, I, I64, I64, I64, P, P, I, I64, P, I, I64, P],
        "ttq_unpack_codes": [P, I64, I64, I, P, P],
        "ttq_status_string": [I],
        "ttq_device_error": [I],
        "ttq_abi_version": [],
        "ttq_codes_ld": [I64, I],
        "ttq_groups_ld": [I64, I],
        "ttq_selftest_bounded_wait": [I, P, P],
        "ttq_channel_moment_total": [P, I64, I64, P, P],
        "ttq_awq_scales_sharded": [P, I64, I64, I64, P, P, P, P, P],
        "ttq_projection_stats_rows": [I64, I64, I64, I],
        "ttq_w_lowbit_gemm_prepared_stats": [P, P, I64, I64, P, P, P, I64, I,
                                             I, P, I, I, P, I, I64, F, P,
                                             I64, P],
        "ttq_stats_reduce": [P, I64, I64, I, P, P],
        "ttq_quantize_gemm_prepared": [P, I, I64, P, P, P, I64, I64, I64, I,
                                       I, P, I, I, P, I, I64, P, P, P, P],
        "ttq_lowrank_factors_workspace_size": [I64, I64, I],
        "ttq_lowrank_factors": [P, I64, I64, I64, P, P, I, I, P, P, P, SZ, P],
        "ttq_lowrank_residual": [P, I64, I64, I64, P, P, I, P, I64, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = I
    lib.ttq_status_string.restype = ctypes.c_char_p
    lib.ttq_w_lowbit_gemm_workspace_size.restype = SZ
    lib.ttq_codes_ld.restype = I64
    lib.ttq_groups_ld.restype = I64
    lib.ttq_projection_stats_rows.restype = I64
    lib.ttq_lowrank_factors_workspace_size.restype = SZ
    return lib


_lib = _load()

# Names the C ABI exports (include/ttq.h).
EXPORTS = ("ttq_act_stats", "ttq_awq_scales", "ttq_act_stats_scales",
           "ttq_quantize_rtn_grouped",
           "ttq_w_lowbit_gemm_workspace_size", "ttq_w_lowbit_gemm",
           "ttq_prepare_activations", "ttq_w_lowbit_gemm_prepared",
           "ttq_lowrank_add", "ttq_unpack_codes", "ttq_status_string",
           "ttq_device_error", "ttq_abi_version", "ttq_codes_ld",
           "ttq_groups_ld", "ttq_selftest_bounded_wait",
           "ttq_channel_moment_total", "ttq_awq_scales_sharded",
           "ttq_projection_stats_rows", "ttq_w_lowbit_gemm_prepared_stats",
           "ttq_stats_reduce", "ttq_quantize_gemm_prepared",
           "ttq_lowrank_factors_workspace_size", "ttq_lowrank_factors",
           "ttq_lowrank_residual")


class _Params(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int), ("group", ctypes.c_int),
                ("alpha", ctypes.c_float), ("lambda_", ctypes.c_float),
                ("p", ctypes.c_float)]


@dataclass(frozen=True)
class TTQParams:
    """Fixed per-layer hyperparameters (Proposed method, bullet 4)."""
    bits: int = 4
    group: int = 128
    alpha: float = 0.5
    lam: float = 0.1
    p: float = 2.0


def _check(status: int, what: str) -> None:
    if status != TTQ_OK:
        raise TTQError(f"{what}: {_lib.ttq_status_string(status).decode()}")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, name: str) -> None:
    """A CUDA tensor on the current device (the one the call launches on)."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TTQError(f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise TTQError(f"{name} is on {t.device}; the call launches on "
                       f"cuda:{cur}")


def _code(t: torch.Tensor, name: str) -> int:
    """The ttq_dtype of a floating tensor."""
    if t.dtype not in _DTYPE:
        raise TTQError(f"{name} must be float32, bfloat16 or float16, not "
                       f"{t.dtype}")
    return _DTYPE[t.dtype]


def _rows(t: torch.Tensor, name: str) -> int:
    """Row pitch (elements) of a 2D tensor whose rows are contiguous."""
    _dev(t, name)
    if t.dim() != 2 or t.stride(1) != 1:
        raise TTQError(f"{name} must be 2D with contiguous rows")
    return t.stride(0)


_CODE_DTYPES = (torch.int32, torch.uint32)


def _buf(t: torch.Tensor, name: str, dtypes, rows: int,
         cols: int | None = None) -> None:
    """A dense device buffer: at least ``rows`` entries ([rows] vector), or
    at least ``rows`` rows of exactly ``cols`` entries."""
    _dev(t, name)
    dtypes = dtypes if isinstance(dtypes, tuple) else (dtypes,)
    if t.dtype not in dtypes:
        raise TTQError(f"{name} must be {' or '.join(map(str, dtypes))}, "
                       f"not {t.dtype}")
    if cols is None:
        ok = t.dim() == 1 and t.numel() >= rows
        want = f"[{rows}]"
    else:
        ok = t.dim() == 2 and t.shape[0] >= rows and t.shape[1] == cols
        want = f"[{rows}, {cols}]"
    if not ok or not t.is_contiguous():
        raise TTQError(f"{name} must be a dense buffer of shape {want}, got "
                       f"{tuple(t.shape)} with strides {t.stride()}")


def _packed(codes, delta, zero, N: int, K: int, bits: int, group: int):
    """Codes, delta and zero of an [N, K] weight in the packed layout."""
    cl, gl = codes_ld(K, bits), groups_ld(K, group)
    if cl <= 0 or gl <= 0:
        raise TTQError(f"no packed layout for K={K}, bits={bits}, "
                       f"group={group}")
    _buf(codes, "codes", _CODE_DTYPES, N, cl)
    _buf(delta, "delta", torch.float32, N, gl)
    _buf(zero, "zero", torch.uint8, N, gl)


def _out(Y: torch.Tensor, name: str, T: int, N: int) -> int:
    """An output [T, N] with contiguous rows; returns its row pitch."""
    ld = _rows(Y, name)
    _code(Y, name)
    if tuple(Y.shape) != (T, N):
        raise TTQError(f"{name} must have shape ({T}, {N}), got "
                       f"{tuple(Y.shape)}")
    return ld


def _factors(A, B, N: int, K: int, dtype) -> int:
    """The low-rank factors A [r, K] and B [N, r] (both or neither);
    returns r."""
    if (A is None) != (B is None):
        raise TTQError("A and B come together")
    if A is None:
        return 0
    r = A.shape[0] if A.dim() == 2 else -1
    _buf(A, "A", dtype, r, K)
    _buf(B, "B", dtype, N, r)
    if B.shape[0] != N:
        raise TTQError(f"B must have {N} rows, got {B.shape[0]}")
    return r


def _ptr(t):
    return None if t is None else t.data_ptr()


def abi_version() -> int:
    return int(_lib.ttq_abi_version())


@functools.lru_cache(maxsize=4096)
def codes_ld(K: int, bits: int) -> int:
    """Row pitch (uint32 words) of the packed codes."""
    return int(_lib.ttq_codes_ld(K, bits))


@functools.lru_cache(maxsize=4096)
def groups_ld(K: int, group: int) -> int:
    """Row pitch (entries) of delta and zero."""
    return int(_lib.ttq_groups_ld(K, group))


def device_error(clear: bool = True) -> int:
    """Sticky device error bits (synchronising read)."""
    return int(_lib.ttq_device_error(1 if clear else 0))


def selftest_bounded_wait(arrive: bool) -> tuple[bool, int]:
    """Runs the kernels' bounded wait on a barrier that completes (arrive)
    or never does. Returns (whether the wait completed, the device error
    bits, which are cleared). Synchronises the device."""
    out = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    _check(_lib.ttq_selftest_bounded_wait(1 if arrive else 0, out.data_ptr(),
                                          _stream()),
           "ttq_selftest_bounded_wait")
    torch.cuda.synchronize()
    done = int(out.item())
    if done not in (0, 1):
        raise TTQError(f"ttq_selftest_bounded_wait wrote {done}")
    return done == 1, device_error(clear=True)


def act_stats(X: torch.Tensor, p: float = 2.0, out: torch.Tensor | None = None,
              accumulate: bool = False) -> torch.Tensor:
    """Step 1: out[j] (+)= sum_t |X[t, j]|^p, fp32 [K]."""
    ldx = _rows(X, "X")
    T, K = X.shape
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=X.device)
    _buf(out, "out", torch.float32, K)
    _check(_lib.ttq_act_stats(X.data_ptr(), _code(X, "X"), T, K, ldx,
                              float(p), 1 if accumulate else 0,
                              out.data_ptr(), _stream()), "ttq_act_stats")
    return out


def awq_scales(sums: torch.Tensor, T_total: int, alpha: float = 0.5,
               lam: float = 0.1, p: float = 2.0, s=None, inv_s=None):
    """Step 2: (s, inv_s) fp32 [K] from the channel sums."""
    _buf(sums, "sums", torch.float32, 0)
    K = sums.shape[0]
    s = torch.empty(K, dtype=torch.float32, device=sums.device) if s is None \
        else s
    inv_s = torch.empty_like(s) if inv_s is None else inv_s
    _buf(s, "s", torch.float32, K)
    _buf(inv_s, "inv_s", torch.float32, K)
    prm = _Params(0, 0, alpha, lam, p)
    _check(_lib.ttq_awq_scales(sums.data_ptr(), int(T_total), K,
                               ctypes.addressof(prm), s.data_ptr(),
                               inv_s.data_ptr(), _stream()), "ttq_awq_scales")
    return s, inv_s


def channel_moment_total(sums: torch.Tensor, T_total: int,
                         out: torch.Tensor | None = None) -> torch.Tensor:
    """sum_j sums[j] / T_total of one shard's channels, fp64 [1] on the
    device (the shard's part of the shrinkage mean)."""
    _buf(sums, "sums", torch.float32, 0)
    K = sums.shape[0]
    out = torch.empty(1, dtype=torch.float64, device=sums.device) \
        if out is None else out
    _buf(out, "out", torch.float64, 1)
    _check(_lib.ttq_channel_moment_total(sums.data_ptr(), int(T_total), K,
                                         out.data_ptr(), _stream()),
           "ttq_channel_moment_total")
    return out


def awq_scales_sharded(sums: torch.Tensor, T_total: int, K_total: int,
                       total: torch.Tensor, alpha: float = 0.5,
                       lam: float = 0.1, p: float = 2.0, s=None, inv_s=None):
    """Step 2 of one shard of the input channels: (s, inv_s) fp32 [K] with
    the shrinkage mean total / K_total, total being the fp64 [1] sum of every
    shard's channel_moment_total."""
    _buf(sums, "sums", torch.float32, 0)
    _buf(total, "total", torch.float64, 1)
    K = sums.shape[0]
    s = torch.empty(K, dtype=torch.float32, device=sums.device) if s is None \
        else s
    inv_s = torch.empty_like(s) if inv_s is None else inv_s
    _buf(s, "s", torch.float32, K)
    _buf(inv_s, "inv_s", torch.float32, K)
    prm = _Params(0, 0, alpha, lam, p)
    _check(_lib.ttq_awq_scales_sharded(sums.data_ptr(), int(T_total), K,
                                       int(K_total), ctypes.addressof(prm),
                                       total.data_ptr(), s.data_ptr(),
                                       inv_s.data_ptr(), _stream()),
           "ttq_awq_scales_sharded")
    return s, inv_s


def new_counter(device=None) -> torch.Tensor:
    """A zeroed device word for act_stats_scales (one per concurrent
    stream; each call leaves it zero again)."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def act_stats_scales(X: torch.Tensor, counter: torch.Tensor,
                     alpha: float = 0.5, lam: float = 0.1, p: float = 2.0,
                     sums=None, s=None, inv_s=None, accumulate: bool = False,
                     T_total: int | None = None):
    """Steps 1 and 2 in one launch: (sums, s, inv_s), each fp32 [K]."""
    ldx = _rows(X, "X")
    _buf(counter, "counter", _CODE_DTYPES, 1)
    T, K = X.shape
    f32 = dict(dtype=torch.float32, device=X.device)
    sums = torch.empty(K, **f32) if sums is None else sums
    s = torch.empty(K, **f32) if s is None else s
    inv_s = torch.empty(K, **f32) if inv_s is None else inv_s
    for t, name in ((sums, "sums"), (s, "s"), (inv_s, "inv_s")):
        _buf(t, name, torch.float32, K)
    prm = _Params(0, 0, alpha, lam, p)
    _check(_lib.ttq_act_stats_scales(
        X.data_ptr(), _code(X, "X"), T, K, ldx, 1 if accumulate else 0,
        int(T if T_total is None else T_total), ctypes.addressof(prm),
        sums.data_ptr(), s.data_ptr(), inv_s.data_ptr(), counter.data_ptr(),
        _stream()), "ttq_act_stats_scales")
    return sums, s, inv_s


def quantize_rtn_grouped(W: torch.Tensor, s: torch.Tensor | None, bits: int,
                         group: int, codes=None, delta=None, zero=None):
    """Step 3: packed codes [N, codes_ld] u32 (held as int32), delta
    [N, groups_ld] fp32, zero [N, groups_ld] u8 (see ttq.h for the layout)."""
    ldw = _rows(W, "W")
    N, K = W.shape
    dev = W.device
    if codes is None:
        codes = torch.empty((N, codes_ld(K, bits)), dtype=torch.int32,
                            device=dev)
    if delta is None:
        delta = torch.empty((N, groups_ld(K, group)), dtype=torch.float32,
                            device=dev)
    if zero is None:
        zero = torch.empty((N, groups_ld(K, group)), dtype=torch.uint8,
                           device=dev)
    if s is not None:
        _buf(s, "s", torch.float32, K)
    _packed(codes, delta, zero, N, K, bits, group)
    _check(_lib.ttq_quantize_rtn_grouped(
        W.data_ptr(), _code(W, "W"), N, K, ldw, _ptr(s), bits, group,
        codes.data_ptr(), delta.data_ptr(), zero.data_ptr(), _stream()),
        "ttq_quantize_rtn_grouped")
    return codes, delta, zero


def workspace_size(T: int, K: int, r: int = 0) -> int:
    return int(_lib.ttq_w_lowbit_gemm_workspace_size(T, K, r))


def w_lowbit_gemm(X: torch.Tensor, inv_s: torch.Tensor, codes: torch.Tensor,
                  delta: torch.Tensor, zero: torch.Tensor, N: int, bits: int,
                  group: int, A: torch.Tensor | None = None,
                  B: torch.Tensor | None = None,
                  out: torch.Tensor | None = None, out_dtype=None,
                  workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Step 4: Y = (X diag(inv_s)) W_hat^T [+ (X A^T) B^T], [T, N]."""
    ldx = _rows(X, "X")
    T, K = X.shape
    r = _factors(A, B, N, K, X.dtype)
    _buf(inv_s, "inv_s", torch.float32, K)
    _packed(codes, delta, zero, N, K, bits, group)
    if out is None:
        out = torch.empty((T, N), dtype=out_dtype or X.dtype, device=X.device)
    ldy = _out(out, "out", T, N)
    need = workspace_size(T, K, r)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _dev(workspace, "workspace")
    if not workspace.is_contiguous():
        raise TTQError("workspace must be contiguous")
    _check(_lib.ttq_w_lowbit_gemm(
        X.data_ptr(), _code(X, "X"), T, K, ldx, inv_s.data_ptr(),
        codes.data_ptr(), delta.data_ptr(), zero.data_ptr(), N, bits, group,
        _ptr(A), _ptr(B), r, out.data_ptr(), _code(out, "out"), ldy,
        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream()), "ttq_w_lowbit_gemm")
    return out


def prepare_activations(X: torch.Tensor, inv_s: torch.Tensor, bits: int,
                        A: torch.Tensor | None = None, Xs=None, U=None):
    """Activation side of step 4: Xs = fp16(X diag(inv_s)) [T, K] (channels
    ordered for `bits`-bit codes, see ttq.h) and, with low-rank factors,
    U = fp16(X A^T) zero-padded to [T, 64]."""
    ldx = _rows(X, "X")
    T, K = X.shape
    r = 0
    if A is not None:
        r = A.shape[0] if A.dim() == 2 else -1
        _buf(A, "A", X.dtype, r, K)
    _buf(inv_s, "inv_s", torch.float32, K)
    if Xs is None:
        Xs = torch.empty((T, K), dtype=torch.float16, device=X.device)
    _buf(Xs, "Xs", torch.float16, T, K)
    if r and U is None:
        U = torch.empty((T, 64), dtype=torch.float16, device=X.device)
    if r:
        _buf(U, "U", torch.float16, T, 64)
    _check(_lib.ttq_prepare_activations(
        X.data_ptr(), _code(X, "X"), T, K, ldx, inv_s.data_ptr(), bits,
        _ptr(A), r, Xs.data_ptr(), _ptr(U) if r else None, _stream()),
        "ttq_prepare_activations")
    return Xs, (U if r else None)


def w_lowbit_gemm_prepared(Xs: torch.Tensor, U: torch.Tensor | None,
                           codes: torch.Tensor, delta: torch.Tensor,
                           zero: torch.Tensor, N: int, bits: int, group: int,
                           B: torch.Tensor | None = None,
                           out: torch.Tensor | None = None,
                           out_dtype=torch.bfloat16) -> torch.Tensor:
    """The projection on prepared operands (one kernel launch; one or two
    tokens run on CUDA cores, more on tensor cores)."""
    _dev(Xs, "Xs")
    if Xs.dim() != 2:
        raise TTQError("Xs must be 2D")
    T, K = Xs.shape
    _buf(Xs, "Xs", torch.float16, T, K)
    r = 0
    if B is not None:
        r = B.shape[1] if B.dim() == 2 else -1
        _buf(B, "B", B.dtype, N, r)
        _code(B, "B")
        if B.shape[0] != N:
            raise TTQError(f"B must have {N} rows, got {B.shape[0]}")
        if U is None:
            raise TTQError("a low-rank projection needs U")
        _buf(U, "U", torch.float16, T, 64)
    _packed(codes, delta, zero, N, K, bits, group)
    if out is None:
        out = torch.empty((T, N), dtype=out_dtype, device=Xs.device)
    ldy = _out(out, "out", T, N)
    _check(_lib.ttq_w_lowbit_gemm_prepared(
        Xs.data_ptr(), _ptr(U) if r else None, T, K, codes.data_ptr(),
        delta.data_ptr(), zero.data_ptr(), N, bits, group, _ptr(B),
        _code(B, "B") if r else 0, r, out.data_ptr(), _code(out, "out"),
        ldy, _stream()), "ttq_w_lowbit_gemm_prepared")
    return out


def quantize_gemm_prepared(W: torch.Tensor, s: torch.Tensor, Xs: torch.Tensor,
                           U: torch.Tensor | None, bits: int, group: int,
                           B: torch.Tensor | None = None,
                           out: torch.Tensor | None = None,
                           out_dtype=torch.bfloat16, store_codes: bool = True,
                           codes=None, delta=None, zero=None):
    """Steps 3 and 4 in one launch (the projection quantizes the bf16 W
    itself): Y [T, N], and (codes, delta, zero) of the quantized weights
    unless store_codes is False (then None)."""
    ldw = _rows(W, "W")
    N, K = W.shape
    _buf(s, "s", torch.float32, K)
    _dev(Xs, "Xs")
    T = Xs.shape[0]
    _buf(Xs, "Xs", torch.float16, T, K)
    r = 0
    if B is not None:
        r = B.shape[1] if B.dim() == 2 else -1
        _buf(B, "B", B.dtype, N, r)
        if B.shape[0] != N:
            raise TTQError(f"B must have {N} rows, got {B.shape[0]}")
        if U is None:
            raise TTQError("a low-rank projection needs U")
        _buf(U, "U", torch.float16, T, 64)
    if store_codes:
        dev = W.device
        cl, gl = codes_ld(K, bits), groups_ld(K, group)
        codes = torch.zeros((N, cl), dtype=torch.int32, device=dev) \
            if codes is None else codes
        delta = torch.zeros((N, gl), dtype=torch.float32, device=dev) \
            if delta is None else delta
        zero = torch.zeros((N, gl), dtype=torch.uint8, device=dev) \
            if zero is None else zero
        _packed(codes, delta, zero, N, K, bits, group)
    if out is None:
        out = torch.empty((T, N), dtype=out_dtype, device=Xs.device)
    ldy = _out(out, "out", T, N)
    _check(_lib.ttq_quantize_gemm_prepared(
        W.data_ptr(), _code(W, "W"), ldw, s.data_ptr(), Xs.data_ptr(),
        _ptr(U) if r else None, T, K, N, bits, group, _ptr(B),
        _code(B, "B") if r else 0, r, out.data_ptr(), _code(out, "out"), ldy,
        _ptr(codes) if store_codes else None,
        _ptr(delta) if store_codes else None,
        _ptr(zero) if store_codes else None, _stream()),
        "ttq_quantize_gemm_prepared")
    return out, ((codes, delta, zero) if store_codes else None)


def projection_stats_rows(T: int, N: int, K: int, bits: int) -> int:
    """Partial rows the fused output statistic needs (0: none for T)."""
    return int(_lib.ttq_projection_stats_rows(T, N, K, bits))


def w_lowbit_gemm_prepared_stats(Xs: torch.Tensor, U: torch.Tensor | None,
                                 codes: torch.Tensor, delta: torch.Tensor,
                                 zero: torch.Tensor, N: int, bits: int,
                                 group: int, B: torch.Tensor | None = None,
                                 p: float = 2.0, out: torch.Tensor | None = None,
                                 out_dtype=torch.bfloat16,
                                 stats: torch.Tensor | None = None):
    """The projection on prepared operands plus the partial statistic of its
    stored output: (Y [T, N], stats [rows, N] fp32); stats_reduce adds the
    rows into the next layer's channel sums."""
    _dev(Xs, "Xs")
    if Xs.dim() != 2:
        raise TTQError("Xs must be 2D")
    T, K = Xs.shape
    _buf(Xs, "Xs", torch.float16, T, K)
    rows = projection_stats_rows(T, N, K, bits)
    if rows == 0:
        raise TTQError(f"no fused statistic for T = {T} (prefill only)")
    r = 0
    if B is not None:
        r = B.shape[1] if B.dim() == 2 else -1
        _buf(B, "B", B.dtype, N, r)
        _code(B, "B")
        if B.shape[0] != N:
            raise TTQError(f"B must have {N} rows, got {B.shape[0]}")
        if U is None:
            raise TTQError("a low-rank projection needs U")
        _buf(U, "U", torch.float16, T, 64)
    _packed(codes, delta, zero, N, K, bits, group)
    if out is None:
        out = torch.empty((T, N), dtype=out_dtype, device=Xs.device)
    ldy = _out(out, "out", T, N)
    if stats is None:
        stats = torch.empty((rows, N), dtype=torch.float32, device=Xs.device)
    _buf(stats, "stats", torch.float32, rows, N)
    if stats.shape[0] != rows:
        raise TTQError(f"stats must have {rows} rows")
    _check(_lib.ttq_w_lowbit_gemm_prepared_stats(
        Xs.data_ptr(), _ptr(U) if r else None, T, K, codes.data_ptr(),
        delta.data_ptr(), zero.data_ptr(), N, bits, group, _ptr(B),
        _code(B, "B") if r else 0, r, out.data_ptr(), _code(out, "out"),
        ldy, float(p), stats.data_ptr(), rows, _stream()),
        "ttq_w_lowbit_gemm_prepared_stats")
    return out, stats


def stats_reduce(partials: torch.Tensor, out: torch.Tensor | None = None,
                 accumulate: bool = False) -> torch.Tensor:
    """out[n] (+)= sum_i partials[i][n], fp32 [N]."""
    _dev(partials, "partials")
    if partials.dim() != 2:
        raise TTQError("partials must be 2D")
    P, N = partials.shape
    _buf(partials, "partials", torch.float32, P, N)
    if out is None:
        out = torch.empty(N, dtype=torch.float32, device=partials.device)
    _buf(out, "out", torch.float32, N)
    _check(_lib.ttq_stats_reduce(partials.data_ptr(), P, N, int(accumulate),
                                 out.data_ptr(), _stream()),
           "ttq_stats_reduce")
    return out


def lowrank_add(X: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                Y: torch.Tensor) -> torch.Tensor:
    """Y += (X A^T) B^T in place."""
    ldx = _rows(X, "X")
    T, K = X.shape
    _dev(B, "B")
    N = B.shape[0]
    r = _factors(A, B, N, K, X.dtype)
    ldy = _out(Y, "Y", T, N)
    _check(_lib.ttq_lowrank_add(X.data_ptr(), _code(X, "X"), T, K, ldx,
                                A.data_ptr(), B.data_ptr(), r, N, Y.data_ptr(),
                                _code(Y, "Y"), ldy, _stream()),
           "ttq_lowrank_add")
    return Y


def lowrank_factors_workspace_size(N: int, K: int, r: int) -> int:
    return int(_lib.ttq_lowrank_factors_workspace_size(N, K, r))


def lowrank_factors(W: torch.Tensor, s: torch.Tensor, omega: torch.Tensor,
                    iters: int = 1, workspace: torch.Tensor | None = None):
    """Per-prompt low-rank factors (B [N, r], A [r, K], bf16) of the bf16
    weight W for the scales s, from the probe vectors omega [r, K] (fp32):
    randomized subspace iteration on W diag(s), B = Q, A = Q^T W."""
    ldw = _rows(W, "W")
    N, K = W.shape
    if W.dtype != torch.bfloat16:
        raise TTQError("W must be bfloat16")
    _buf(s, "s", torch.float32, K)
    if omega.dim() != 2 or omega.shape[1] != K:
        raise TTQError(f"omega must be [r, {K}], got {tuple(omega.shape)}")
    r = omega.shape[0]
    _buf(omega, "omega", torch.float32, r, K)
    need = lowrank_factors_workspace_size(N, K, r)
    if need == 0:
        raise TTQError(f"no factor workspace for N={N}, K={K}, r={r}")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _buf(workspace, "workspace", torch.uint8, need)
    B = torch.empty((N, r), dtype=torch.bfloat16, device=W.device)
    A = torch.empty((r, K), dtype=torch.bfloat16, device=W.device)
    _check(_lib.ttq_lowrank_factors(W.data_ptr(), N, K, ldw, s.data_ptr(),
                                    omega.data_ptr(), r, int(iters),
                                    B.data_ptr(), A.data_ptr(),
                                    workspace.data_ptr(), workspace.numel(),
                                    _stream()), "ttq_lowrank_factors")
    return B, A


def lowrank_residual(W: torch.Tensor, B: torch.Tensor, A: torch.Tensor,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """R = bf16(W - B A) (bf16 W [N, K], B [N, r], A [r, K])."""
    ldw = _rows(W, "W")
    N, K = W.shape
    if W.dtype != torch.bfloat16:
        raise TTQError("W must be bfloat16")
    r = _factors(A, B, N, K, torch.bfloat16)
    if out is None:
        out = torch.empty((N, K), dtype=torch.bfloat16, device=W.device)
    ldr = _out(out, "out", N, K)
    if out.dtype != torch.bfloat16:
        raise TTQError("out must be bfloat16")
    _check(_lib.ttq_lowrank_residual(W.data_ptr(), N, K, ldw, B.data_ptr(),
                                     A.data_ptr(), r, out.data_ptr(), ldr,
                                     _stream()), "ttq_lowrank_residual")
    return out


def unpack_codes(codes: torch.Tensor, K: int, bits: int) -> torch.Tensor:
    """One uint8 per weight, [N, K]."""
    _dev(codes, "codes")
    N = codes.shape[0]
    _buf(codes, "codes", _CODE_DTYPES, N, codes_ld(K, bits))
    q = torch.empty((N, K), dtype=torch.uint8, device=codes.device)
    _check(_lib.ttq_unpack_codes(codes.data_ptr(), N, K, bits, q.data_ptr(),
                                 _stream()), "ttq_unpack_codes")
    return q


class TTQLinear:
    """One linear layer run the TTQ way: per prompt, statistics and scales
    (one launch) -> quantize -> low-bit projection (+ optional static
    low-rank term).

    ``W`` is the stored weight ([N, K], or the residual W - B A when ``A`` and
    ``B`` are given). Buffers are allocated once per (T) and reused; the
    layer's arrival counter makes concurrent use of one layer object on
    several streams unsafe (use one object per stream).
    """

    def __init__(self, W: torch.Tensor, params: TTQParams, A=None, B=None):
        self.W, self.A, self.B, self.prm = W, A, B, params
        N, K = W.shape
        dev = W.device
        self.sums = torch.empty(K, dtype=torch.float32, device=dev)
        self.s = torch.empty(K, dtype=torch.float32, device=dev)
        self.inv_s = torch.empty(K, dtype=torch.float32, device=dev)
        self.counter = new_counter(dev)
        self.codes = torch.empty((N, codes_ld(K, params.bits)),
                                 dtype=torch.int32, device=dev)
        gl = groups_ld(K, params.group)
        self.delta = torch.empty((N, gl), dtype=torch.float32, device=dev)
        self.zero = torch.empty((N, gl), dtype=torch.uint8, device=dev)
        self._ws = None

    def calibrate(self, X: torch.Tensor) -> None:
        """Online statistics and quantization from this prompt's input."""
        p = self.prm
        act_stats_scales(X, self.counter, p.alpha, p.lam, p.p, self.sums,
                         self.s, self.inv_s)
        quantize_rtn_grouped(self.W, self.s, p.bits, p.group, self.codes,
                             self.delta, self.zero)

    def project(self, X: torch.Tensor, out: torch.Tensor | None = None):
        T, K = X.shape
        r = 0 if self.A is None else self.A.shape[0]
        need = workspace_size(T, K, r)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=X.device)
        return w_lowbit_gemm(X, self.inv_s, self.codes, self.delta, self.zero,
                             self.W.shape[0], self.prm.bits, self.prm.group,
                             self.A, self.B, out=out, workspace=self._ws)

    def __call__(self, X: torch.Tensor, out: torch.Tensor | None = None):
        self.calibrate(X)
        return self.project(X, out)
