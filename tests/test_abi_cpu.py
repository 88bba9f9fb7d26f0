"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/ttq.h declares, and rejects bad arguments before
touching the device. Also checks that the oracle and the CUDA path share no
code."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttq.h")
LIB = os.path.join(ROOT, "test_weight_quantization_b200", "libttq.so")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from test_weight_quantization_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ttq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_hot_path():
    names = declared_functions()
    for n in ("ttq_act_stats", "ttq_awq_scales", "ttq_quantize_rtn_grouped",
              "ttq_w_lowbit_gemm", "ttq_lowrank_add"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    lib.ttq_status_string.restype = ctypes.c_char_p
    assert lib.ttq_status_string(0) == b"TTQ_OK"
    assert lib.ttq_status_string(1) == b"TTQ_ERR_INVALID_ARG"
    assert lib.ttq_status_string(99) == b"TTQ_ERR_UNKNOWN"
    assert lib.ttq_abi_version() == 8


def test_workspace_size(lib):
    f = lib.ttq_w_lowbit_gemm_workspace_size
    f.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    f.restype = ctypes.c_size_t
    assert f(16, 4096, 0) >= 16 * 4096 * 2
    assert f(16, 4096, 16) >= f(16, 4096, 0) + 16 * 64 * 2
    assert f(0, 4096, 0) == 0


def test_bad_arguments_are_rejected_before_launch(lib):
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: checks fail first
    lib.ttq_selftest_bounded_wait.argtypes = [I, P, P]
    assert lib.ttq_selftest_bounded_wait(0, None, None) == 1
    assert lib.ttq_selftest_bounded_wait(1, ctypes.c_void_p(0x100002),
                                         None) == 1  # misaligned
    lib.ttq_act_stats.argtypes = [P, I, I64, I64, I64, F, I, P, P]
    assert lib.ttq_act_stats(None, 1, 8, 64, 64, 2.0, 0, fake, None) == 1
    assert lib.ttq_act_stats(fake, 1, 8, 60, 64, 2.0, 0, fake, None) == 1  # K%8
    assert lib.ttq_act_stats(fake, 1, 8, 64, 64, -1.0, 0, fake, None) == 1
    assert lib.ttq_act_stats(fake, 7, 8, 64, 64, 2.0, 0, fake, None) == 1
    f = lib.ttq_act_stats_scales
    f.argtypes = [P, I, I64, I64, I64, I, I64, P, P, P, P, P, P]

    class Prm(ctypes.Structure):
        _fields_ = [("bits", I), ("group", I), ("alpha", F), ("lambda_", F),
                    ("p", F)]
    prm = Prm(0, 0, 0.5, 0.1, 2.0)
    pp = ctypes.addressof(prm)
    assert f(fake, 1, 8, 64, 64, 0, 8, pp, fake, fake, fake, None, None) == 1
    assert f(fake, 1, 8, 64, 64, 0, 7, pp, fake, fake, fake, fake, None) == 1
    assert f(fake, 1, 8, 64, 64, 2, 8, pp, fake, fake, fake, fake, None) == 1
    assert f(fake, 1, 8, 64, 64, 0, 8, None, fake, fake, fake, fake, None) == 1
    # overlapping outputs are refused (s holds partials during the launch)
    base = 0x200000
    same = ctypes.c_void_p(base)
    assert f(fake, 1, 8, 64, 64, 0, 8, pp, same, same, ctypes.c_void_p(base + 4096),
             ctypes.c_void_p(base + 8192), None) == 1
    assert f(fake, 1, 8, 64, 64, 0, 8, pp, ctypes.c_void_p(base),
             ctypes.c_void_p(base + 128), ctypes.c_void_p(base + 4096),
             ctypes.c_void_p(base + 8192), None) == 1  # s starts inside sums
    assert f(fake, 1, 8, 64, 64, 0, 8, pp, ctypes.c_void_p(base),
             ctypes.c_void_p(base + 4096), ctypes.c_void_p(base + 8192),
             ctypes.c_void_p(base + 4096 + 16), None) == 1  # counter in s
    bad = Prm(0, 0, 0.5, 1.5, 2.0)
    assert f(fake, 1, 8, 64, 64, 0, 8, ctypes.addressof(bad), fake, fake, fake,
             fake, None) == 1
    lib.ttq_quantize_rtn_grouped.argtypes = [P, I, I64, I64, I64, P, I, I, P,
                                             P, P, P]
    q = lib.ttq_quantize_rtn_grouped
    assert q(fake, 1, 4, 64, 64, None, 9, 32, fake, fake, fake, None) == 1
    assert q(fake, 1, 4, 64, 64, None, 4, 24, fake, fake, fake, None) == 1
    assert q(fake, 1, 4, 48, 48, None, 4, 16, fake, fake, fake, None) == 1
    lib.ttq_w_lowbit_gemm.argtypes = [P, I, I64, I64, I64, P, P, P, P, I64, I,
                                      I, P, P, I, P, I, I64, P, ctypes.c_size_t,
                                      P]
    g = lib.ttq_w_lowbit_gemm
    # workspace too small
    assert g(fake, 1, 16, 64, 64, fake, fake, fake, fake, 32, 4, 32, None,
             None, 0, fake, 1, 32, fake, 16, None) == 1
    # low-rank rank without factors
    assert g(fake, 1, 16, 64, 64, fake, fake, fake, fake, 32, 4, 32, None,
             None, 8, fake, 1, 32, fake, 1 << 20, None) == 1
    lib.ttq_unpack_codes.argtypes = [P, I64, I64, I, P, P]
    assert lib.ttq_unpack_codes(None, 4, 64, 4, fake, None) == 1
    SZ = ctypes.c_size_t
    ws = lib.ttq_lowrank_factors_workspace_size
    ws.argtypes = [I64, I64, I]
    ws.restype = SZ
    assert ws(256, 512, 16) > 0 and ws(256, 512, 0) == 0
    assert ws(256, 512, 65) == 0
    lf = lib.ttq_lowrank_factors
    lf.argtypes = [P, I64, I64, I64, P, P, I, I, P, P, P, SZ, P]
    big = 1 << 30
    a16 = ctypes.c_void_p(0x1000000)     # 16-byte aligned, never touched
    Bp, Ap = ctypes.c_void_p(0x2000000), ctypes.c_void_p(0x3000000)
    wsp = ctypes.c_void_p(0x4000000)
    need = ws(256, 512, 16)
    assert lf(a16, 256, 512, 512, a16, a16, 0, 1, Bp, Ap, wsp, big,
              None) == 1                                  # r = 0
    assert lf(a16, 256, 512, 512, a16, a16, 16, 17, Bp, Ap, wsp, big,
              None) == 1                                  # iters > 16
    assert lf(a16, 256, 512, 500, a16, a16, 16, 1, Bp, Ap, wsp, big,
              None) == 1                                  # ldw < K
    assert lf(a16, 256, 512, 516, a16, a16, 16, 1, Bp, Ap, wsp, big,
              None) == 1                                  # ldw % 8
    assert lf(ctypes.c_void_p(0x1000008), 256, 512, 512, a16, a16, 16, 1, Bp,
              Ap, wsp, big, None) == 1                    # W not 16-aligned
    assert lf(a16, 256, 512, 512, a16, a16, 16, 1, Bp, Ap, wsp, need - 1,
              None) == 1                                  # workspace short
    assert lf(a16, 256, 512, 512, a16, a16, 16, 1, Bp, Ap,
              ctypes.c_void_p(0x4000080), big, None) == 1  # ws not 256-aligned
    assert lf(a16, 256, 512, 512, a16, a16, 16, 1, Bp,
              ctypes.c_void_p(0x2000000 + 256 * 16), wsp, big,
              None) == 1                                  # A overlaps B
    lr = lib.ttq_lowrank_residual
    lr.argtypes = [P, I64, I64, I64, P, P, I, P, I64, P]
    Rp = ctypes.c_void_p(0x5000000)
    assert lr(a16, 64, 512, 512, Bp, Ap, 0, Rp, 512, None) == 1   # r = 0
    assert lr(a16, 64, 512, 512, Bp, Ap, 65, Rp, 512, None) == 1  # r > 64
    assert lr(a16, 64, 512, 512, Bp, Ap, 16, Rp, 508, None) == 1  # ldr < K
    assert lr(a16, 64, 512, 512, Bp, Ap, 16,
              ctypes.c_void_p(0x1000000 + 1024), 512, None) == 1  # R inside W
    assert lr(a16, 64, 512, 512, Bp, Ap, 16, a16, 520, None) == 1  # W, other ld


def test_oracle_and_cuda_path_share_no_code():
    csrc = glob.glob(os.path.join(ROOT, "test_weight_quantization_b200",
                                  "**", "*.*"), recursive=True)
    for path in csrc:
        if path.endswith((".cu", ".cuh", ".h", ".py")):
            text = open(path, errors="ignore").read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), \
                path
            assert "ttq_oracle" not in text, path
    osrc = open(os.path.join(ROOT, "oracle", "ttq_oracle.c")).read()
    includes = re.findall(r"^\s*#\s*include\s*[<\"]([^>\"]+)", osrc, re.M)
    assert all(i in ("math.h", "stdint.h", "stdlib.h", "string.h")
               for i in includes), includes
    opy = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    assert "test_weight_quantization_b200" not in opy


def test_packed_pitches(lib):
    lib.ttq_codes_ld.argtypes = [ctypes.c_int64, ctypes.c_int]
    lib.ttq_codes_ld.restype = ctypes.c_int64
    lib.ttq_groups_ld.argtypes = [ctypes.c_int64, ctypes.c_int]
    lib.ttq_groups_ld.restype = ctypes.c_int64
    assert lib.ttq_codes_ld(768, 3) == 72        # 72 words, already aligned
    assert lib.ttq_codes_ld(96, 3) == 12         # 9 words padded to 12
    assert lib.ttq_codes_ld(4096, 4) == 512
    assert lib.ttq_groups_ld(768, 32) == 32      # 24 groups padded to 32
    assert lib.ttq_groups_ld(4096, 128) == 32
    assert lib.ttq_groups_ld(48, 16) == 16
    assert lib.ttq_codes_ld(100, 3) == 0 and lib.ttq_groups_ld(96, 24) == 0


def test_empty_inputs_are_refused_before_launch(lib):
    """T = 0, N = 0 or K = 0 is an invalid argument for every call (the
    header requires T, N >= 1 and K a positive multiple of 32 or 8); nothing
    is launched, so fake pointers are never touched."""
    P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    fake = ctypes.c_void_p(0x100000)
    st = lib.ttq_act_stats
    st.argtypes = [P, I, I64, I64, I64, F, I, P, P]
    assert st(fake, 1, 0, 64, 64, 2.0, 0, fake, None) == 1
    assert st(fake, 1, 8, 0, 64, 2.0, 0, fake, None) == 1
    q = lib.ttq_quantize_rtn_grouped
    q.argtypes = [P, I, I64, I64, I64, P, I, I, P, P, P, P]
    assert q(fake, 1, 0, 64, 64, None, 4, 32, fake, fake, fake, None) == 1
    assert q(fake, 1, 4, 0, 64, None, 4, 32, fake, fake, fake, None) == 1
    pr = lib.ttq_prepare_activations
    pr.argtypes = [P, I, I64, I64, I64, P, I, P, I, P, P, P]
    assert pr(fake, 1, 0, 64, 64, fake, 4, None, 0, fake, None, None) == 1
    gp = lib.ttq_w_lowbit_gemm_prepared
    gp.argtypes = [P, P, I64, I64, P, P, P, I64, I, I, P, I, I, P, I, I64, P]
    assert gp(fake, None, 0, 64, fake, fake, fake, 32, 4, 32, None, 1, 0,
              fake, 1, 32, None) == 1
    assert gp(fake, None, 4, 64, fake, fake, fake, 0, 4, 32, None, 1, 0,
              fake, 1, 32, None) == 1
    lr = lib.ttq_lowrank_add
    lr.argtypes = [P, I, I64, I64, I64, P, P, I, I64, P, I, I64, P]
    assert lr(fake, 1, 0, 64, 64, fake, fake, 16, 32, fake, 1, 32, None) == 1
    un = lib.ttq_unpack_codes
    un.argtypes = [P, I64, I64, I, P, P]
    assert un(fake, 0, 64, 4, fake, None) == 1


def test_binding_refuses_host_tensors_and_bad_layouts():
    """The Python binding checks its tensors before calling the library:
    host tensors and rows that are not contiguous raise TTQError."""
    import torch
    from test_weight_quantization_b200 import ttq
    X = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ttq.TTQError):
        ttq.act_stats(X)
    with pytest.raises(ttq.TTQError):
        ttq.quantize_rtn_grouped(X, None, 4, 32)
    with pytest.raises(ttq.TTQError):
        ttq.act_stats_scales(X, torch.zeros(1, dtype=torch.int32))


@pytest.mark.parametrize("K", [32, 96, 768, 4096, 11008])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
def test_row_pitches_match_the_documented_formulas(lib, K, bits):
    """ttq_codes_ld: K*bits/32 words rounded up to 4; ttq_groups_ld: K/g
    entries rounded up to 16 (16-byte rows for TMA)."""
    from test_weight_quantization_b200 import ttq
    words = K * bits // 32
    assert ttq.codes_ld(K, bits) == (words + 3) // 4 * 4
    for g in (16, 32, 64, 128):
        if K % g == 0:
            assert ttq.groups_ld(K, g) == (K // g + 15) // 16 * 16


def _no_cuda_device():
    import torch
    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_cuda_device(),
                    reason="its control calls would launch on fake pointers")
def test_packed_operands_must_be_16_byte_aligned(lib):
    """The projection reads codes, delta and zero with 16-byte and
    tensor-memory-accelerator loads: a pointer off a 16-byte boundary is an
    invalid argument for every projection entry point. Each refused call
    differs from an accepted one only in that pointer (the accepted control
    cannot launch here: this host has no CUDA device)."""
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    ok = 0x100000
    g = lib.ttq_w_lowbit_gemm
    g.argtypes = [P, I, I64, I64, I64, P, P, P, P, I64, I, I, P, P, I, P, I,
                  I64, P, ctypes.c_size_t, P]
    gp = lib.ttq_w_lowbit_gemm_prepared
    gp.argtypes = [P, P, I64, I64, P, P, P, I64, I, I, P, I, I, P, I, I64, P]
    na = lib.ttq_w_lowbit_gemm_noalloc
    na.argtypes = [P, I, I64, I64, I64, P, P, P, P, I64, I, I, P, P, I, P, I,
                   I64, P]

    def calls(c, d, z):
        return (
            g(ok, 1, 16, 64, 64, ok, c, d, z, 32, 4, 32, None, None, 0, ok, 1,
              32, ok, 1 << 20, None),
            gp(ok, None, 4, 64, c, d, z, 32, 4, 32, None, 1, 0, ok, 1, 32,
               None),
            na(ok, 1, 16, 64, 64, ok, c, d, z, 32, 4, 32, None, None, 0, ok,
               1, 32, None))
    assert all(st != 1 for st in calls(ok, ok, ok))
    for off in (4, 8):
        for c, d, z in ((ok + off, ok, ok), (ok, ok + off, ok),
                        (ok, ok, ok + off)):
            assert calls(c, d, z) == (1, 1, 1), (off, c, d, z)


@pytest.mark.skipif(not _no_cuda_device(),
                    reason="an accepted call would launch on fake pointers")
def test_sizes_beyond_the_index_range_are_refused(lib):
    """The largest sizes each entry point accepts: 32-bit block and row
    counts. One past them is an invalid argument, refused before launch
    (these pointers are never dereferenced)."""
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    ok = 0x100000
    big = 1 << 31
    q = lib.ttq_quantize_rtn_grouped
    q.argtypes = [P, I, I64, I64, I64, P, I, I, P, P, P, P]
    # N * (K / 32) blocks must stay below 2^31
    assert q(ok, 1, big // 2, 64, 64, None, 4, 32, ok, ok, ok, None) == 1
    g = lib.ttq_w_lowbit_gemm
    g.argtypes = [P, I, I64, I64, I64, P, P, P, P, I64, I, I, P, P, I, P, I,
                  I64, P, ctypes.c_size_t, P]
    assert g(ok, 1, big, 64, 64, ok, ok, ok, ok, 32, 4, 32, None, None, 0, ok,
             1, 32, ok, 1 << 62, None) == 1                       # T
    assert g(ok, 1, 16, 64, 64, ok, ok, ok, ok, big, 4, 32, None, None, 0, ok,
             1, big, ok, 1 << 20, None) == 1                      # N
    gp = lib.ttq_w_lowbit_gemm_prepared
    gp.argtypes = [P, P, I64, I64, P, P, P, I64, I, I, P, I, I, P, I, I64, P]
    assert gp(ok, None, big, 64, ok, ok, ok, 32, 4, 32, None, 1, 0, ok, 1, 32,
              None) == 1
    assert gp(ok, None, 4, 64, ok, ok, ok, big, 4, 32, None, 1, 0, ok, 1, big,
              None) == 1
    pr = lib.ttq_prepare_activations
    pr.argtypes = [P, I, I64, I64, I64, P, I, P, I, P, P, P]
    # T * (K / 16) spans must stay below 2^31
    assert pr(ok, 1, big // 4, 64, 64, ok, 4, None, 0, ok, None, None) == 1
