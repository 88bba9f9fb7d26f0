"""The Python binding's argument checks, on the host: every documented call
pattern passes them and reaches the C ABI with the right pitches and dtype
codes, and buffers of the wrong dtype, shape, density or device are refused
before the library is called. The library is replaced by a recorder and the
device check by one that accepts host tensors, so no kernel runs."""
import pytest
import torch

from test_weight_quantization_b200 import ttq


class Recorder:
    """Stands in for libttq: records each call and returns TTQ_OK."""

    def __init__(self, real):
        self.real, self.calls = real, []

    def __getattr__(self, name):
        if name in ("ttq_codes_ld", "ttq_groups_ld",
                    "ttq_w_lowbit_gemm_workspace_size", "ttq_status_string"):
            return getattr(self.real, name)

        def call(*args):
            self.calls.append((name, args))
            return ttq.TTQ_OK
        return call


@pytest.fixture
def rec(monkeypatch):
    r = Recorder(ttq._lib)
    monkeypatch.setattr(ttq, "_lib", r)
    monkeypatch.setattr(ttq, "_stream", lambda: 0)

    def host_dev(t, name):
        if not isinstance(t, torch.Tensor):
            raise ttq.TTQError(f"{name} must be a tensor")
    monkeypatch.setattr(ttq, "_dev", host_dev)
    # tensors the binding allocates with device="cuda" are made on the host
    real_empty = torch.empty

    def empty(*a, device=None, **k):
        return real_empty(*a, **k)
    monkeypatch.setattr(ttq.torch, "empty", empty)
    return r


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16, torch.float16])
def test_documented_call_patterns_pass(rec, dt):
    T, K, N, r, b, g = 40, 256, 96, 16, 4, 32
    X = torch.zeros(T, K, dtype=dt)
    sums = ttq.act_stats(X)
    assert rec.calls[-1][0] == "ttq_act_stats"
    assert rec.calls[-1][1][1] == ttq._DTYPE[dt]
    # a view with a row pitch, accumulated into a given buffer
    big = torch.zeros(T, K + 64, dtype=dt)
    ttq.act_stats(big[:, :K], out=sums, accumulate=True)
    assert rec.calls[-1][1][4] == K + 64  # ldx
    s, inv = ttq.awq_scales(sums, T)
    ttq.awq_scales(sums, T, 0.5, 0.1, 2.0, s, inv)
    ctr = torch.zeros(1, dtype=torch.int32)
    ttq.act_stats_scales(X, ctr)
    ttq.act_stats_scales(X, ctr, 0.5, 0.1, 2.0, sums, s, inv, True, 2 * T)
    W = torch.zeros(N, K, dtype=dt)
    c, d, z = ttq.quantize_rtn_grouped(W, s, b, g)
    assert c.shape == (N, ttq.codes_ld(K, b)) and c.dtype == torch.int32
    assert d.shape == z.shape == (N, ttq.groups_ld(K, g))
    ttq.quantize_rtn_grouped(W, None, b, g, c, d, z)
    A = torch.zeros(r, K, dtype=dt)
    B = torch.zeros(N, r, dtype=dt)
    for out_dtype in (None, torch.float32, torch.bfloat16, torch.float16):
        Y = ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, out_dtype=out_dtype)
        assert Y.shape == (T, N)
        ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, A, B)
    pitched = torch.zeros(T, N + 24, dtype=torch.bfloat16)[:, :N]
    ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, out=pitched)
    assert rec.calls[-1][1][17] == N + 24  # ldy
    ws = torch.zeros(ttq.workspace_size(T, K), dtype=torch.uint8)
    ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, workspace=ws)
    Xs, U = ttq.prepare_activations(X, inv, b)
    assert U is None and Xs.dtype == torch.float16
    Xs2, U2 = ttq.prepare_activations(X, inv, b, A)
    assert U2.shape == (T, 64)
    ttq.prepare_activations(X, inv, b, None, Xs)
    ttq.prepare_activations(X, inv, b, A, Xs2, U2)
    ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, N, b, g)
    ttq.w_lowbit_gemm_prepared(Xs2, U2, c, d, z, N, b, g, B, out_dtype=dt)
    ttq.w_lowbit_gemm_prepared(Xs[:2], None, c, d, z, N, b, g,
                               out=torch.zeros(2, N, dtype=torch.bfloat16))
    # stacked weights: more code rows than one projection uses
    ttq.w_lowbit_gemm_prepared(Xs, None, c[: N // 2], d[: N // 2],
                               z[: N // 2], N // 2, b, g)
    ttq.lowrank_add(X, A, B, torch.zeros(T, N, dtype=dt))
    ttq.unpack_codes(c, K, b)
    layer = ttq.TTQLinear(W, ttq.TTQParams(b, g), A, B)
    layer(X)
    names = [n for n, _ in rec.calls]
    for n in ("ttq_act_stats", "ttq_awq_scales", "ttq_act_stats_scales",
              "ttq_quantize_rtn_grouped", "ttq_w_lowbit_gemm",
              "ttq_prepare_activations", "ttq_w_lowbit_gemm_prepared",
              "ttq_lowrank_add", "ttq_unpack_codes"):
        assert n in names


def test_bad_buffers_are_refused_before_the_library(rec):
    T, K, N, b, g = 8, 128, 32, 4, 32
    X = torch.zeros(T, K, dtype=torch.bfloat16)
    W = torch.zeros(N, K, dtype=torch.bfloat16)
    sums, s, inv = f32(K), f32(K), f32(K)
    c, d, z = ttq.quantize_rtn_grouped(W, s, b, g)
    A, B = torch.zeros(4, K, dtype=torch.bfloat16), \
        torch.zeros(N, 4, dtype=torch.bfloat16)
    Xs, U = ttq.prepare_activations(X, inv, b, A)
    before = len(rec.calls)
    bad = [
        lambda: ttq.act_stats(X, out=f32(K - 1)),                 # short
        lambda: ttq.act_stats(X, out=torch.zeros(K, dtype=torch.float64)),
        lambda: ttq.act_stats(X.to(torch.float64)),               # dtype
        lambda: ttq.act_stats(X.t()),                             # layout
        lambda: ttq.awq_scales(sums, T, s=f32(K)[::2]),           # strided
        lambda: ttq.act_stats_scales(X, torch.zeros(1, dtype=torch.float32)),
        lambda: ttq.act_stats_scales(X, torch.zeros(1, dtype=torch.int32),
                                     s=f32(K - 8)),
        lambda: ttq.quantize_rtn_grouped(W, f32(K - 32), b, g),
        lambda: ttq.quantize_rtn_grouped(W, s, b, g, c[:, :-1], d, z),
        lambda: ttq.quantize_rtn_grouped(W, s, b, g, c, d.double(), z),
        lambda: ttq.quantize_rtn_grouped(W, s, b, g, c, d, z[: N - 1]),
        lambda: ttq.quantize_rtn_grouped(W, s, 9, g),             # no layout
        lambda: ttq.w_lowbit_gemm(X, inv, c, d, z, N + 1, b, g),  # rows
        lambda: ttq.w_lowbit_gemm(X, inv, c, d, z, N, 3, g),      # width
        lambda: ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, A),   # no B
        lambda: ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g, A,
                                  B.float()),                     # B dtype
        lambda: ttq.w_lowbit_gemm(X, inv, c, d, z, N, b, g,
                                  out=torch.zeros(T, N + 1)),     # out shape
        lambda: ttq.w_lowbit_gemm(X, inv[:K - 1], c, d, z, N, b, g),
        lambda: ttq.prepare_activations(X, inv, b, None,
                                        torch.zeros(T, K)),      # Xs dtype
        lambda: ttq.prepare_activations(X, inv, b, A, Xs,
                                        torch.zeros(T, 32,
                                                    dtype=torch.float16)),
        lambda: ttq.w_lowbit_gemm_prepared(Xs.float(), None, c, d, z, N, b,
                                           g),
        lambda: ttq.w_lowbit_gemm_prepared(Xs, None, c, d, z, N, b, g, B),
        lambda: ttq.w_lowbit_gemm_prepared(Xs, U, c, d, z, N, b, g,
                                           B[: N - 1]),
        lambda: ttq.lowrank_add(X, A, B, torch.zeros(T, N + 1,
                                                     dtype=torch.bfloat16)),
        lambda: ttq.lowrank_add(X, A[:, :K - 8], B,
                                torch.zeros(T, N, dtype=torch.bfloat16)),
        lambda: ttq.unpack_codes(c[:, :-1], K, b),
    ]
    for i, fn in enumerate(bad):
        with pytest.raises(ttq.TTQError):
            fn()
        assert len(rec.calls) == before, f"case {i} reached the library"
