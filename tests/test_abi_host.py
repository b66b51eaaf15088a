"""The C-ABI library on the host: it loads, exports every symbol the header
declares, rejects bad arguments before touching the GPU, and its host layout
helpers agree with the oracle.  No compute call runs here (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import build as zt_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zt_q4.h")


@pytest.fixture(scope="module")
def zt():
    zt_build.build()
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def declared_symbols(path):
    text = open(path).read()
    return sorted(set(re.findall(r"ZT_API\s+[\w\s\*]*?\b(zt_\w+)\s*\(", text)))


def test_header_declares_the_abi():
    syms = declared_symbols(HEADER)
    for want in ("zt_q4_gemv", "zt_q4_gate_up_silu", "zt_q4_lmhead_argmax",
                 "zt_q4_lmhead_workspace_bytes", "zt_q4_pack_host", "zt_q4_unpack_host",
                 "zt_q4_strerror", "zt_q4_version",
                 "zt_q4_last_cuda_error"):
        assert want in syms


def test_library_exports_every_declared_symbol(zt):
    for path in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if path.endswith(".h"):
            for sym in declared_symbols(os.path.join(ROOT, "include", path)):
                assert hasattr(zt.lib, sym), f"{sym} declared in {path} but not exported"


def test_strerror_and_version(zt):
    for code in (0, -1, -2, -3, -4, -5, -6, 12345):
        assert isinstance(zt.strerror(code), str) and zt.strerror(code)
    assert zt.version()[0] == 1


FAKE = 0x10000  # 64 KiB-aligned fake address: never dereferenced (checks fail first)


@pytest.mark.parametrize("fn", ["zt_q4_gemv", "zt_q4_gate_up_silu"])
def test_bad_arguments_rejected(zt, fn):
    f = getattr(zt.lib, fn)
    ok = (FAKE, FAKE, FAKE, FAKE)
    # null pointers
    for i in range(4):
        ptrs = list(ok)
        ptrs[i] = None
        assert f(*ptrs, 1, 64, 64, None) == zt.ZT_ERR_INVALID_ARG
    # shapes
    for M, N, K in ((0, 64, 64), (17, 64, 64), (-1, 64, 64), (1, 0, 64), (1, 64, 0),
                    (1, 64, 16), (1, 64, 48), (1, 64, 100), (1, -5, 64)):
        assert f(*ok, M, N, K, None) == zt.ZT_ERR_INVALID_ARG, (M, N, K)
    # misalignment: qw and x need 16 bytes, scales and y 2
    assert f(FAKE + 8, FAKE, FAKE, FAKE, 1, 64, 64, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE + 1, FAKE, FAKE, 1, 64, 64, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE + 4, FAKE, 1, 64, 64, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE + 1, 1, 64, 64, None) == zt.ZT_ERR_MISALIGNED


def test_gate_up_row_count_overflow(zt):
    assert zt.lib.zt_q4_gate_up_silu(FAKE, FAKE, FAKE, FAKE, 1, 2**30 + 1, 64, None) == zt.ZT_ERR_INVALID_ARG


def test_lmhead_arguments(zt):
    f = zt.lib.zt_q4_lmhead_argmax
    ws = zt.lmhead_workspace_bytes(1, 1000, 256)
    assert ws > 0
    assert zt.lmhead_workspace_bytes(0, 1000, 256) == 0
    assert zt.lmhead_workspace_bytes(1, 1000, 100) == 0
    assert zt.lmhead_workspace_bytes(16, 1000, 256) >= ws
    assert zt.lmhead_workspace_bytes(1, 10, 256) == zt.lmhead_workspace_bytes(1, 10**6, 8192)
    args = [FAKE] * 6
    for i in range(6):
        a = list(args)
        a[i] = None
        assert f(*a, ws, 1, 1000, 256, None) == zt.ZT_ERR_INVALID_ARG
    assert f(*args, ws - 1, 1, 1000, 256, None) == zt.ZT_ERR_WORKSPACE
    assert f(*args, 0, 1, 1000, 256, None) == zt.ZT_ERR_WORKSPACE
    a = list(args)
    a[3] = FAKE + 2          # logits need 4 bytes
    assert f(*a, ws, 1, 1000, 256, None) == zt.ZT_ERR_MISALIGNED
    a = list(args)
    a[5] = FAKE + 8          # workspace needs 16
    assert f(*a, ws, 1, 1000, 256, None) == zt.ZT_ERR_MISALIGNED
    assert f(*args, ws, 17, 1000, 256, None) == zt.ZT_ERR_INVALID_ARG


def test_pack_unpack_host_matches_oracle(zt, oracle):
    g = np.random.default_rng(21)
    qw = g.integers(0, 2**32, size=(13, 40), dtype=np.uint32)
    q = zt.unpack_host(qw, 320)
    assert np.array_equal(q, oracle.unpack(qw, 320))
    assert np.array_equal(zt.pack_host(q), qw)
    assert np.array_equal(zt.pack_host(q), oracle.pack(q))


def test_pack_host_rejects_codes_above_15(zt):
    q = np.zeros((2, 16), dtype=np.uint8)
    q[1, 5] = 16
    with pytest.raises(zt.ZtError):
        zt.pack_host(q)
    rc = zt.lib.zt_q4_pack_host(None, 2, 16, None)
    assert rc == zt.ZT_ERR_INVALID_ARG


def test_pass_arguments_rejected(zt):
    P = zt.ZtProj
    ok = P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0)
    arr = (P * 1)(ok)
    ws = zt.lib.zt_q4_pass_workspace_bytes(arr, 1, 1)
    assert ws > 0
    f = zt.lib.zt_q4_pass
    assert f(None, 1, 1, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(arr, 0, 1, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(arr, zt.ZT_Q4_PASS_MAX + 1, 1, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(arr, 1, 17, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(arr, 1, 1, None, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(arr, 1, 1, FAKE, ws - 1, None) == zt.ZT_ERR_WORKSPACE
    assert f(arr, 1, 1, FAKE + 8, ws, None) == zt.ZT_ERR_MISALIGNED
    for bad in (P(FAKE, FAKE, FAKE, FAKE, None, 7, 64, 64, 0),              # unknown kind
                P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_LM_HEAD, 64, 64, 0),  # LM head without argmax
                P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 48, 0),     # K % 32
                P(None, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0)):
        assert f((P * 2)(ok, bad), 2, 1, FAKE, 1 << 20, None) == zt.ZT_ERR_INVALID_ARG
    mis = P(FAKE, FAKE, FAKE + 8, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0)
    assert f((P * 1)(mis), 1, 1, FAKE, ws, None) == zt.ZT_ERR_MISALIGNED
    lm = P(FAKE, FAKE, FAKE, FAKE, FAKE, zt.ZT_Q4_LM_HEAD, 64, 64, 0)
    assert zt.lib.zt_q4_pass_workspace_bytes((P * 2)(ok, lm), 2, 1) > ws
    assert zt.lib.zt_q4_pass_errors(None, 1, None) == zt.ZT_ERR_INVALID_ARG


def test_pass_norm_arguments_rejected(zt):
    """The add + RMSNorm prologue's checks run before any launch."""
    import ctypes
    P, Nm = zt.ZtProj, zt.ZtNorm
    f = zt.lib.zt_q4_pass

    def call(nm, x=None):
        proj = P(FAKE, FAKE, x, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0, norm=ctypes.pointer(nm) if nm else None)
        return f((P * 1)(proj), 1, 1, FAKE, 1 << 20, None)

    for bad in (Nm(None, None, FAKE, None, None, 1e-5),                 # no residual
                Nm(FAKE, None, None, None, None, 1e-5),                 # no gamma
                Nm(FAKE, None, FAKE, None, None, -1e-5),               # negative eps
                Nm(FAKE, None, FAKE, None, None, float("nan")),
                Nm(FAKE, None, FAKE, None, None, float("inf")),
                Nm(FAKE, None, FAKE, FAKE + 64, None, 1e-5),            # residual_out overlaps residual
                Nm(FAKE, FAKE + 4096, FAKE, FAKE + 4096 + 112, None, 1e-5)):   # ... overlaps delta
        assert call(bad) == zt.ZT_ERR_INVALID_ARG
    for bad in (Nm(FAKE + 2, None, FAKE, None, None, 1e-5),
                Nm(FAKE, FAKE + 8, FAKE, None, None, 1e-5),
                Nm(FAKE, None, FAKE + 8, None, None, 1e-5),
                Nm(FAKE, None, FAKE, FAKE + 4100, None, 1e-5),
                Nm(FAKE, None, FAKE, None, FAKE + 2, 1e-5)):
        assert call(bad) == zt.ZT_ERR_MISALIGNED
    # without a prologue x is required
    assert call(None, x=None) == zt.ZT_ERR_INVALID_ARG


def test_pass_rope_and_ld_out_arguments_rejected(zt):
    """RoPE epilogue and output-stride checks run before any launch."""
    import ctypes
    P, R = zt.ZtProj, zt.ZtRope
    f = zt.lib.zt_q4_pass

    def call(rope, kind=zt.ZT_Q4_GEMV, N=96, ld_out=0, argmax=None):
        proj = P(FAKE, FAKE, FAKE, FAKE, argmax, kind, N, 64, 0, ld_out, rope=ctypes.pointer(rope) if rope else None)
        return f((P * 1)(proj), 1, 1, FAKE, 1 << 20, None)

    good = R(FAKE, 32, 10000.0)
    for bad in (R(None, 32, 10000.0),             # no positions
                R(FAKE, 33, 10000.0),             # odd head_dim
                R(FAKE, 64, 10000.0),             # N % head_dim != 0
                R(FAKE, 0, 10000.0),
                R(FAKE, 32, 0.0), R(FAKE, 32, -2.0), R(FAKE, 32, float("nan")), R(FAKE, 32, float("inf"))):
        assert call(bad) == zt.ZT_ERR_INVALID_ARG
    assert call(good, kind=zt.ZT_Q4_GATE_UP_SILU) == zt.ZT_ERR_INVALID_ARG       # RoPE is for plain projections
    assert call(good, kind=zt.ZT_Q4_LM_HEAD, argmax=FAKE) == zt.ZT_ERR_INVALID_ARG
    assert call(R(FAKE + 2, 32, 10000.0)) == zt.ZT_ERR_MISALIGNED
    assert call(None, ld_out=95) == zt.ZT_ERR_INVALID_ARG                         # stride below N


def test_pass_group_size_rejected(zt):
    """Groups other than 32, 64, 128 (0 = 32), or not dividing K, fail before any launch."""
    P = zt.ZtProj
    f = zt.lib.zt_q4_pass
    for group, K in ((16, 256), (96, 384), (256, 512), (128, 320), (64, 96)):
        proj = P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, K, 0, 0, group)
        assert f((P * 1)(proj), 1, 1, FAKE, 1 << 20, None) == zt.ZT_ERR_INVALID_ARG, (group, K)


# ------------------------------------------------- batched prefill (M > 16) --
def test_prefill_symbols_declared():
    syms = declared_symbols(HEADER)
    for want in ("zt_q4_dequant_f16", "zt_q4_gemm_f16w", "zt_q4_gemm_f16w_workspace_bytes", "zt_q4_gemm_f16w_errors",
                 "zt_q4_gemm", "zt_q4_gemm_workspace_bytes", "zt_q4_gemm_errors"):
        assert want in syms


def test_gemm_workspace_bytes(zt):
    """The plan (and so the workspace) is a function of the shape alone."""
    f, g = zt.lib.zt_q4_gemm_workspace_bytes, zt.lib.zt_q4_gemm_f16w_workspace_bytes
    w16 = ((9216 * 3072 * 2 + 255) // 256) * 256
    assert g(512, 9216, 3072) == 256                      # one wave of 256 x 128 tiles: no split
    assert f(512, 9216, 3072) == w16 + 256
    assert g(4096, 16384, 3072) == 256                    # 256 x 256 tiles, many waves
    assert g(512, 3072, 8192) == 256 + 3 * 512 * 3072 * 4  # 36 tiles: 3 splits of fp32 partials
    assert g(128, 9216, 8192) == 256 + 4 * 128 * 9216 * 4
    assert g(40, 3072, 8192) == 256 + 6 * 40 * 3072 * 4    # weight rows as A: 24 tiles, 6 splits
    assert g(512, 3072, 512) == 256                       # K too short to split
    assert f(3, 3, 32) == 256 + 256
    assert f(0, 9216, 3072) == 0 and f(8, 8, 48) == 0 and f(8, 0, 32) == 0 and g(1, 8, 0) == 0
    for M, N, K in ((17, 128, 64), (300, 640, 2048), (2048, 3072, 8192)):
        assert f(M, N, K) == ((N * K * 2 + 255) // 256) * 256 + g(M, N, K)
        assert (g(M, N, K) - 256) % (M * N * 4) == 0 and (g(M, N, K) - 256) // (M * N * 4) <= 8


def test_gemm_arguments_rejected(zt):
    """Every check runs before a launch: these calls touch no device memory."""
    g = zt.lib.zt_q4_gemm
    ws = zt.gemm_workspace_bytes(40, 256, 64)
    ok = [FAKE, FAKE, FAKE, FAKE, 40, 256, 64, 32, FAKE, ws, None]

    def call(**kw):
        a = list(ok)
        names = ["qw", "scales", "x", "y", "M", "N", "K", "group", "ws", "ws_bytes", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return g(*a)

    for k in ("qw", "scales", "x", "y", "ws"):
        assert call(**{k: None}) == zt.ZT_ERR_INVALID_ARG
    assert call(M=0) == zt.ZT_ERR_INVALID_ARG
    assert call(M=(1 << 22) + 1) == zt.ZT_ERR_INVALID_ARG
    assert call(N=0) == zt.ZT_ERR_INVALID_ARG
    assert call(K=48) == zt.ZT_ERR_INVALID_ARG
    assert call(group=48) == zt.ZT_ERR_INVALID_ARG
    assert call(group=128) == zt.ZT_ERR_INVALID_ARG          # K = 64 is not a multiple of 128
    assert call(qw=FAKE + 8) == zt.ZT_ERR_MISALIGNED
    assert call(x=FAKE + 8) == zt.ZT_ERR_MISALIGNED
    assert call(ws=FAKE + 8) == zt.ZT_ERR_MISALIGNED
    assert call(scales=FAKE + 1) == zt.ZT_ERR_MISALIGNED
    assert call(y=FAKE + 1) == zt.ZT_ERR_MISALIGNED
    assert call(ws_bytes=ws - 1) == zt.ZT_ERR_WORKSPACE


def test_dequant_and_gemm_f16w_arguments_rejected(zt):
    d = zt.lib.zt_q4_dequant_f16
    assert d(None, FAKE, FAKE, 8, 64, 32, None) == zt.ZT_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE, 8, 48, 32, None) == zt.ZT_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE, 8, 64, 16, None) == zt.ZT_ERR_INVALID_ARG
    assert d(FAKE, FAKE, FAKE + 8, 8, 64, 32, None) == zt.ZT_ERR_MISALIGNED
    assert d(FAKE + 4, FAKE, FAKE, 8, 64, 32, None) == zt.ZT_ERR_MISALIGNED
    f = zt.lib.zt_q4_gemm_f16w
    ws = zt.gemm_f16w_workspace_bytes(17, 64, 64)
    assert f(FAKE, FAKE, FAKE, 17, 64, 64, None, ws, None) == zt.ZT_ERR_INVALID_ARG     # no workspace
    assert f(FAKE, FAKE, FAKE, 0, 64, 64, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert f(FAKE + 8, FAKE, FAKE, 17, 64, 64, FAKE, ws, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, 17, 64, 64, FAKE + 8, ws, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, 17, 64, 64, FAKE, ws - 1, None) == zt.ZT_ERR_WORKSPACE
    out = ctypes.c_uint(0)
    assert zt.lib.zt_q4_gemm_errors(None, 8, 64, ctypes.byref(out)) == zt.ZT_ERR_INVALID_ARG
    assert zt.lib.zt_q4_gemm_f16w_errors(None, ctypes.byref(out)) == zt.ZT_ERR_INVALID_ARG


def test_withhold_hook_needs_a_wait(zt):
    """The error-path test hook refuses a list without waits (nothing to expire)."""
    P = zt.ZtProj
    arr = (P * 2)(P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0),
                  P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0))
    assert zt.lib.zt_q4_pass_test_withhold(arr, 2, 1, FAKE, 1 << 20, None) == zt.ZT_ERR_INVALID_ARG
    assert zt.lib.zt_q4_pass_test_withhold(None, 2, 1, FAKE, 1 << 20, None) == zt.ZT_ERR_INVALID_ARG


def test_checked_build_hooks(zt):
    """The default library is not the checked build and refuses its test hook before any
    CUDA call; the checked library (where built) says so, loads, and exports the same ABI."""
    import ctypes
    P = zt.ZtProj
    arr = (P * 1)(P(FAKE, FAKE, FAKE, FAKE, None, zt.ZT_Q4_GEMV, 64, 64, 0))
    assert not zt.is_checked_build()
    assert zt.lib.zt_q4_pass_test_cut(arr, 1, 1, FAKE, 1 << 20, None, 3) == zt.ZT_ERR_UNSUPPORTED
    if not os.path.exists(zt.CHECKED_LIB_PATH):
        pytest.skip("libzt_q4_checked.so not built")
    lib = ctypes.CDLL(zt.CHECKED_LIB_PATH)
    assert lib.zt_q4_build_flags() == 1
    for sym in declared_symbols(HEADER):
        assert hasattr(lib, sym), sym
    lib.zt_q4_pass_test_cut.argtypes = [ctypes.POINTER(P), ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int]
    assert lib.zt_q4_pass_test_cut(arr, 1, 1, FAKE, 1 << 20, None, 0) == zt.ZT_ERR_INVALID_ARG


def test_gemm_gate_up_arguments(zt):
    f = zt.lib.zt_q4_gemm_gate_up_workspace_bytes
    assert f(512, 8192, 3072) == ((2 * 8192 * 3072 * 2 + 255) // 256) * 256 + 256
    assert f(0, 8192, 3072) == 0 and f(8, 0, 3072) == 0 and f(8, 8, 48) == 0 and f(8, 2 ** 30 + 1, 32) == 0
    g = zt.lib.zt_q4_gemm_gate_up_silu
    ws = f(40, 256, 512)
    assert g(None, FAKE, FAKE, FAKE, 40, 256, 512, 32, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert g(FAKE, FAKE, FAKE, FAKE, 40, 256, 512, 48, FAKE, ws, None) == zt.ZT_ERR_INVALID_ARG
    assert g(FAKE, FAKE, FAKE + 8, FAKE, 40, 256, 512, 32, FAKE, ws, None) == zt.ZT_ERR_MISALIGNED
    assert g(FAKE, FAKE, FAKE, FAKE, 40, 256, 512, 32, FAKE, ws - 1, None) == zt.ZT_ERR_WORKSPACE
    h = zt.lib.zt_q4_gemm_f16w_gate_up_silu
    assert h(FAKE, FAKE, FAKE, 40, 256, 512, None, 256, None) == zt.ZT_ERR_INVALID_ARG
    assert h(FAKE, FAKE, FAKE, 40, 256, 512, FAKE, 255, None) == zt.ZT_ERR_WORKSPACE
    assert h(FAKE + 8, FAKE, FAKE, 40, 256, 512, FAKE, 256, None) == zt.ZT_ERR_MISALIGNED


def test_gemm_grid_limit_rejected_before_launch(zt):
    """Weight-row tiles beyond CUDA's 65535 grid rows: ZT_ERR_UNSUPPORTED from
    the host checks (no device needed); a large but legal shape passes them
    (and only then meets the device: ZT_ERR_DEVICE without a GPU)."""
    import torch
    M, K = 128, 32
    for N in (20_000_000,):            # > 65535 tiles of even 256 weight rows
        ws = zt.gemm_workspace_bytes(M, N, K)
        assert zt.lib.zt_q4_gemm(FAKE, FAKE, FAKE, FAKE, M, N, K, 32, FAKE, ws, None) == zt.ZT_ERR_UNSUPPORTED
        gws = zt.gemm_f16w_workspace_bytes(M, N, K)
        assert zt.lib.zt_q4_gemm_f16w(FAKE, FAKE, FAKE, M, N, K, FAKE, gws, None) == zt.ZT_ERR_UNSUPPORTED
    N = 9_000_000
    ws = zt.gemm_gate_up_workspace_bytes(M, N, K)
    assert zt.lib.zt_q4_gemm_gate_up_silu(FAKE, FAKE, FAKE, FAKE, M, N, K, 32, FAKE, ws, None) == zt.ZT_ERR_UNSUPPORTED
    assert zt.lib.zt_q4_gemm_f16w_gate_up_silu(FAKE, FAKE, FAKE, M, N, K, FAKE, 256, None) == zt.ZT_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        N = 32064                                   # the Phi-3-mini LM head: legal
        ws = zt.gemm_workspace_bytes(M, N, K)
        assert zt.lib.zt_q4_gemm(FAKE, FAKE, FAKE, FAKE, M, N, K, 32, FAKE, ws, None) == zt.ZT_ERR_DEVICE


# ------------------------------------------------ decode launch plan --
def test_decode_plan_covers_every_small_batch_shape(zt):
    """Every decode shape with M <= 16 has a plan, from the shapes alone: the
    activations are staged whole while they fit in shared memory, and in K
    windows (multiples of one 256-k item) beyond; more than 8 tokens that
    would need windows run as two column blocks.  No device is touched."""
    for M in range(1, 17):
        for K in (32, 256, 1056, 3072, 4096, 8192, 11008, 12320, 16384, 40000, 65536, 131072, 1 << 20):
            for n in (1, 4, 129, 192):
                cps, stages, kw, cb, warps = zt.pass_plan(M, K, n)
                assert cps in (1, 2) and 2 <= stages <= 4, (M, K, n)
                assert warps == 8 or (warps == 16 and cps == 1 and kw == 0), (M, K, n, warps)
                assert kw == 0 or (kw % 256 == 0 and 256 <= kw < K), (M, K, n, kw)
                assert cb == 1 or (cb == 2 and M > 8), (M, K, n, cb)
                if M > 8 and cb == 1:
                    assert kw == 0, (M, K, n)   # 16 columns are never windowed


def test_decode_plan_pins(zt):
    """Where the plan switches, on the shapes of the benchmark and its configs."""
    # the benchmark's Phi-3-mini pass at M = 1: x staged whole, one CTA of 16 warps per SM, 4-deep rings;
    # a single projection of one token: two CTAs of 8 warps per SM
    assert zt.pass_plan(1, 8192, 129) == (1, 4, 0, 1, 16)
    assert zt.pass_plan(1, 3072, 1) == (2, 4, 0, 1, 8) and zt.pass_plan(2, 3072, 1)[4] == 16
    # config 3 (gate_up K = 3072) at M = 16 still fits whole, 16 warps with 2-deep rings, one column block
    assert zt.pass_plan(16, 3072, 1) == (1, 2, 0, 1, 16)
    # M = 8 with K = 8192: x (131 KB) leaves room for 16 warps' rings 2 deep, with the least
    # partial buffer; M = 9 (16 columns, 262 KB of x at whole K) needs 8 warps
    assert zt.pass_plan(8, 8192, 129) == (1, 2, 0, 1, 16)
    assert zt.pass_plan(9, 8192, 1)[4] == 8
    # Llama-7B down (K = 11008): whole at M = 4, windows from M = 8, and two column blocks
    # of windows at M = 16
    assert zt.pass_plan(4, 11008, 1)[2] == 0
    assert zt.pass_plan(8, 11008, 1)[2:] == (2816, 1, 8)
    assert zt.pass_plan(16, 11008, 1)[2:] == (2816, 2, 8)
    # Phi-3 down (8192): 16 columns fit whole up to M = 9; at M = 12 and 16 two column
    # blocks of at most 8 tokens, each whole
    assert zt.pass_plan(9, 8192, 1)[2:4] == (0, 1)
    assert zt.pass_plan(12, 8192, 1)[2:4] == (0, 2) and zt.pass_plan(16, 8192, 129)[2:4] == (0, 2)
    # single token: 16 warps (paired layout, 144 staged bytes per group of 32) up to K ~ 30000,
    # then 8 warps (plain layout, 80 bytes per group) whole up to K ~ 72000, windows beyond
    assert zt.pass_plan(1, 16384, 129)[2:] == (0, 1, 16)
    assert zt.pass_plan(1, 32768, 129)[2:] == (0, 1, 8)
    assert zt.pass_plan(1, 65536, 1)[2] == 0
    assert zt.pass_plan(1, 98304, 1)[2] > 0 and zt.pass_plan(1, 131072, 1)[2] > 0
    # windows go with two CTAs per SM
    assert zt.pass_plan(16, 16384, 192)[0] == 2


def test_decode_plan_rejects_bad_shapes(zt):
    c = ctypes.c_int(0)
    for M, K, n in ((0, 256, 1), (17, 256, 1), (1, 16, 1), (1, 100, 1), (1, 256, 0), (1, 256, 193)):
        assert zt.lib.zt_q4_pass_plan(M, K, n, *[ctypes.byref(c)] * 5) == zt.ZT_ERR_INVALID_ARG
    assert zt.lib.zt_q4_pass_plan(1, 256, 1, None, *[ctypes.byref(c)] * 4) == zt.ZT_ERR_INVALID_ARG
    assert zt.lib.zt_q4_pass_plan(1, 256, 1, *[ctypes.byref(c)] * 4, None) == zt.ZT_ERR_INVALID_ARG


def test_noalloc_misaligned_rejected_without_cuda(zt):
    """The allocation-free LM head checks alignment before its first CUDA call
    (on this host without a GPU it would otherwise report a device error)."""
    f = zt.lib.zt_q4_lmhead_argmax_noalloc
    assert f(FAKE + 4, FAKE, FAKE, FAKE, FAKE, 1, 100, 256, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE + 1, FAKE, FAKE, FAKE, 1, 100, 256, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE + 8, FAKE, FAKE, 1, 100, 256, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE + 2, FAKE, 1, 100, 256, None) == zt.ZT_ERR_MISALIGNED
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 1, 100, 256, None) == zt.ZT_ERR_MISALIGNED
