"""Thin ctypes binding of ``libzt_q4.so`` (declared in ``include/zt_q4.h``).

Argument marshalling only: torch supplies device memory and the current CUDA
stream; every step of the computation runs in the library's kernels.  Importing
this module loads the library and fails loudly when it is missing -- there is
no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# ZT_Q4_LIB names another build of the same library to load instead, e.g. the
# bounds-checked libzt_q4_checked.so beside this file
LIB_PATH = os.environ.get("ZT_Q4_LIB") or os.path.join(_PKG, "libzt_q4.so")
CHECKED_LIB_PATH = os.path.join(_PKG, "libzt_q4_checked.so")
ZT_Q4_ERR_BOUNDS = 2

ZT_OK = 0
ZT_ERR_INVALID_ARG = -1
ZT_ERR_MISALIGNED = -2
ZT_ERR_WORKSPACE = -3
ZT_ERR_LAUNCH = -4
ZT_ERR_UNSUPPORTED = -5
ZT_ERR_DEVICE = -6

_P = ctypes.c_void_p
_I = ctypes.c_int


class ZtError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        cuda = lib.zt_q4_last_cuda_error().decode() if status in (ZT_ERR_LAUNCH, ZT_ERR_DEVICE) else ""
        super().__init__(f"{what}: status {status}: {strerror(status)}" + (f" [{cuda}]" if cuda else ""))


ZT_Q4_GEMV = 0
ZT_Q4_GATE_UP_SILU = 1
ZT_Q4_LM_HEAD = 2
ZT_Q4_PASS_MAX = 192


class ZtNorm(ctypes.Structure):
    """struct zt_q4_norm of include/zt_q4.h (residual add + RMSNorm prologue)"""
    _fields_ = [("residual", ctypes.c_void_p), ("delta", ctypes.c_void_p), ("gamma", ctypes.c_void_p),
                ("residual_out", ctypes.c_void_p), ("x_out", ctypes.c_void_p), ("eps", ctypes.c_float)]


class ZtRope(ctypes.Structure):
    """struct zt_q4_rope of include/zt_q4.h (rotary position embedding epilogue)"""
    _fields_ = [("pos", ctypes.c_void_p), ("head_dim", ctypes.c_int), ("theta", ctypes.c_float)]


class ZtProj(ctypes.Structure):
    """struct zt_q4_proj of include/zt_q4.h"""
    _fields_ = [("qw", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("x", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("argmax", ctypes.c_void_p), ("kind", ctypes.c_int),
                ("N", ctypes.c_int), ("K", ctypes.c_int), ("wait", ctypes.c_int), ("ld_out", ctypes.c_int),
                ("group", ctypes.c_int), ("norm", ctypes.POINTER(ZtNorm)), ("rope", ctypes.POINTER(ZtRope))]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m int4_group_quantized_q4f16_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.zt_q4_gemv.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P]
    lib.zt_q4_gate_up_silu.argtypes = [_P, _P, _P, _P, _I, _I, _I, _P]
    lib.zt_q4_lmhead_workspace_bytes.argtypes = [_I, _I, _I]
    lib.zt_q4_lmhead_workspace_bytes.restype = ctypes.c_size_t
    lib.zt_q4_lmhead_argmax.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _P]
    lib.zt_q4_lmhead_argmax_noalloc.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _P]
    lib.zt_q4_lmhead_argmax_noalloc.restype = ctypes.c_int
    lib.zt_q4_pass_workspace_bytes.argtypes = [ctypes.POINTER(ZtProj), _I, _I]
    lib.zt_q4_pass_workspace_bytes.restype = ctypes.c_size_t
    lib.zt_q4_pass.argtypes = [ctypes.POINTER(ZtProj), _I, _I, _P, ctypes.c_size_t, _P]
    lib.zt_q4_pass.restype = ctypes.c_int
    lib.zt_q4_pass_errors.argtypes = [_P, _I, ctypes.POINTER(ctypes.c_uint)]
    lib.zt_q4_pass_plan.argtypes = [_I, _I, _I] + [ctypes.POINTER(_I)] * 5
    lib.zt_q4_pass_plan.restype = ctypes.c_int
    lib.zt_q4_pass_test_withhold.argtypes = [ctypes.POINTER(ZtProj), _I, _I, _P, ctypes.c_size_t, _P]
    lib.zt_q4_pass_test_withhold.restype = ctypes.c_int
    lib.zt_q4_pass_test_cut.argtypes = [ctypes.POINTER(ZtProj), _I, _I, _P, ctypes.c_size_t, _P, _I]
    lib.zt_q4_pass_test_cut.restype = ctypes.c_int
    lib.zt_q4_build_flags.argtypes = []
    lib.zt_q4_build_flags.restype = ctypes.c_int
    lib.zt_q4_pass_errors.restype = ctypes.c_int
    lib.zt_q4_dequant_f16.argtypes = [_P, _P, _P, _I, _I, _I, _P]
    lib.zt_q4_gemm_f16w.argtypes = [_P, _P, _P, _I, _I, _I, _P, ctypes.c_size_t, _P]
    lib.zt_q4_gemm_f16w_workspace_bytes.argtypes = [_I, _I, _I]
    lib.zt_q4_gemm_f16w_workspace_bytes.restype = ctypes.c_size_t
    lib.zt_q4_gemm_f16w_errors.argtypes = [_P, ctypes.POINTER(ctypes.c_uint)]
    lib.zt_q4_gemm_workspace_bytes.argtypes = [_I, _I, _I]
    lib.zt_q4_gemm_workspace_bytes.restype = ctypes.c_size_t
    lib.zt_q4_gemm.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P, ctypes.c_size_t, _P]
    lib.zt_q4_gemm_errors.argtypes = [_P, _I, _I, ctypes.POINTER(ctypes.c_uint)]
    lib.zt_q4_gemm_gate_up_workspace_bytes.argtypes = [_I, _I, _I]
    lib.zt_q4_gemm_gate_up_workspace_bytes.restype = ctypes.c_size_t
    lib.zt_q4_gemm_gate_up_silu.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P, ctypes.c_size_t, _P]
    lib.zt_q4_gemm_f16w_gate_up_silu.argtypes = [_P, _P, _P, _I, _I, _I, _P, ctypes.c_size_t, _P]
    for f in (lib.zt_q4_dequant_f16, lib.zt_q4_gemm_f16w, lib.zt_q4_gemm, lib.zt_q4_gemm_errors,
              lib.zt_q4_gemm_f16w_errors, lib.zt_q4_gemm_gate_up_silu, lib.zt_q4_gemm_f16w_gate_up_silu):
        f.restype = ctypes.c_int
    lib.zt_q4_pack_host.argtypes = [_P, _I, _I, _P]
    lib.zt_q4_unpack_host.argtypes = [_P, _I, _I, _P]
    lib.zt_q4_strerror.argtypes = [_I]
    lib.zt_q4_strerror.restype = ctypes.c_char_p
    lib.zt_q4_version.argtypes = []
    lib.zt_q4_last_cuda_error.argtypes = []
    lib.zt_q4_last_cuda_error.restype = ctypes.c_char_p
    for f in (lib.zt_q4_gemv, lib.zt_q4_gate_up_silu, lib.zt_q4_lmhead_argmax,
              lib.zt_q4_pack_host, lib.zt_q4_unpack_host, lib.zt_q4_version):
        f.restype = ctypes.c_int
    return lib


lib = _load()


def strerror(status: int) -> str:
    return lib.zt_q4_strerror(int(status)).decode()


def version() -> Tuple[int, int]:
    v = lib.zt_q4_version()
    return v >> 16, v & 0xFFFF


def is_checked_build() -> bool:
    """True when the loaded library is the bounds-checked build (-DZT_Q4_CHECKED)."""
    return bool(lib.zt_q4_build_flags() & 1)


def _check(rc: int, what: str) -> None:
    if rc != ZT_OK:
        raise ZtError(rc, what)


# ------------------------------------------------------------ host layout --
def pack_host(q: np.ndarray) -> np.ndarray:
    """codes uint8 [N][K] (0..15) -> packed uint32 [N][K/8], low nibble first."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    N, K = q.shape
    qw = np.empty((N, K // 8), dtype=np.uint32)
    _check(lib.zt_q4_pack_host(q.ctypes.data, N, K, qw.ctypes.data), "zt_q4_pack_host")
    return qw


def unpack_host(qw: np.ndarray, K: int) -> np.ndarray:
    qw = np.ascontiguousarray(qw, dtype=np.uint32)
    N = qw.shape[0]
    q = np.empty((N, K), dtype=np.uint8)
    _check(lib.zt_q4_unpack_host(qw.ctypes.data, N, K, q.ctypes.data), "zt_q4_unpack_host")
    return q


# ---------------------------------------------------------- device calls --
def _torch():
    import torch
    return torch


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dims(qw, scales, x, rows_mult: int, group: int = 32):
    torch = _torch()
    for t, name in ((qw, "qw"), (scales, "scales"), (x, "x")):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if qw.dtype not in (torch.int32, torch.uint32):
        raise TypeError("qw must hold 32-bit words (int32 or uint32)")
    if scales.dtype != torch.float16 or x.dtype != torch.float16:
        raise TypeError("scales and x must be float16")
    x2 = x if x.dim() == 2 else x.view(1, -1)
    M, K = x2.shape
    n_rows = qw.shape[0]
    if qw.dim() != 2 or qw.shape[1] * 8 != K or K % group or scales.shape != (n_rows, K // group):
        raise ValueError(f"shape mismatch: qw {tuple(qw.shape)}, scales {tuple(scales.shape)}, x {tuple(x.shape)}")
    if n_rows % rows_mult:
        raise ValueError("gate/up weights need an even number of rows")
    return M, n_rows // rows_mult, K


def gemv(qw, scales, x, y=None, stream=None):
    """y[M][N] fp16 = dequant(qw, scales) @ x^T (torch CUDA tensors)."""
    torch = _torch()
    M, N, K = _dims(qw, scales, x, 1)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check(lib.zt_q4_gemv(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(),
                          M, N, K, _stream_handle(stream)), "zt_q4_gemv")
    return y


def gate_up_silu(qw, scales, x, y=None, stream=None):
    """y[M][N] fp16 = SiLU(gate . x) * (up . x); qw has 2N rows, gate first."""
    torch = _torch()
    M, N, K = _dims(qw, scales, x, 2)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _check(lib.zt_q4_gate_up_silu(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(),
                                  M, N, K, _stream_handle(stream)), "zt_q4_gate_up_silu")
    return y


# ------------------------------------------------- batched prefill (M > 16) --
def _group_of(K: int, scales) -> int:
    g = K // scales.shape[1]
    if g * scales.shape[1] != K:
        raise ValueError("scales must have K / group columns")
    return g


def dequant_f16(qw, scales, w16=None, stream=None):
    """w16 fp16 [N][K] = fp16((q - 7) * s), one rounding to nearest even."""
    torch = _torch()
    N, K = qw.shape[0], qw.shape[1] * 8
    g = _group_of(K, scales)
    _dims(qw, scales, torch.empty((1, K), dtype=torch.float16, device=qw.device), 1, g)
    if w16 is None:
        w16 = torch.empty((N, K), dtype=torch.float16, device=qw.device)
    _check(lib.zt_q4_dequant_f16(qw.data_ptr(), scales.data_ptr(), w16.data_ptr(), N, K, g,
                                 _stream_handle(stream)), "zt_q4_dequant_f16")
    return w16


def gemm_f16w_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.zt_q4_gemm_f16w_workspace_bytes(M, N, K))


def gemm_f16w(w16, x, y=None, workspace=None, stream=None):
    """y fp16 [M][N] = x [M][K] @ w16^T on the tensor cores; workspace: uint8
    CUDA tensor of gemm_f16w_workspace_bytes(M, N, K) bytes (error word and
    split-K partials)."""
    torch = _torch()
    for t, name in ((w16, "w16"), (x, "x")):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float16 or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous 2-D float16 CUDA tensor")
    (N, K), M = w16.shape, x.shape[0]
    if x.shape[1] != K:
        raise ValueError("x and w16 disagree on K")
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = torch.empty((gemm_f16w_workspace_bytes(M, N, K),), dtype=torch.uint8, device=x.device)
    _check(lib.zt_q4_gemm_f16w(w16.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, workspace.data_ptr(),
                               workspace.numel(), _stream_handle(stream)), "zt_q4_gemm_f16w")
    return y


def gemm_f16w_errors(workspace) -> int:
    out = ctypes.c_uint(0)
    _check(lib.zt_q4_gemm_f16w_errors(workspace.data_ptr(), ctypes.byref(out)), "zt_q4_gemm_f16w_errors")
    return int(out.value)


def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.zt_q4_gemm_workspace_bytes(M, N, K))


def gemm(qw, scales, x, y=None, workspace=None, stream=None):
    """Batched prefill: y fp16 [M][N] = x @ fp16(dequant(qw, scales))^T: the
    dequant into the workspace, then the tensor-core GEMM (and, for shapes
    split along K, the ordered sum of the partials)."""
    torch = _torch()
    N, K = qw.shape[0], qw.shape[1] * 8
    g = _group_of(K, scales)
    M, _, _ = _dims(qw, scales, x, 1, g)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = torch.empty((gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device=x.device)
    _check(lib.zt_q4_gemm(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, g,
                          workspace.data_ptr(), workspace.numel(), _stream_handle(stream)), "zt_q4_gemm")
    return y


def gemm_errors(workspace, N: int, K: int) -> int:
    out = ctypes.c_uint(0)
    _check(lib.zt_q4_gemm_errors(workspace.data_ptr(), N, K, ctypes.byref(out)), "zt_q4_gemm_errors")
    return int(out.value)


def gemm_gate_up_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.zt_q4_gemm_gate_up_workspace_bytes(M, N, K))


def gemm_gate_up_silu(qw, scales, x, y=None, workspace=None, stream=None):
    """Batched fused FFN: y fp16 [M][N] = SiLU(x @ W16_gate^T) * (x @ W16_up^T),
    qw / scales with 2N rows (gate first), through the binary16 weights."""
    torch = _torch()
    two_n, K = qw.shape[0], qw.shape[1] * 8
    g = _group_of(K, scales)
    M, N, _ = _dims(qw, scales, x, 2, g)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = torch.empty((gemm_gate_up_workspace_bytes(M, N, K),), dtype=torch.uint8, device=x.device)
    _check(lib.zt_q4_gemm_gate_up_silu(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K, g,
                                       workspace.data_ptr(), workspace.numel(), _stream_handle(stream)),
           "zt_q4_gemm_gate_up_silu")
    return y


def gemm_f16w_gate_up_silu(w16, x, y=None, workspace=None, stream=None):
    """The fused FFN on binary16 weights w16 [2N][K] (gate rows first)."""
    torch = _torch()
    for t, name in ((w16, "w16"), (x, "x")):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float16 or t.dim() != 2:
            raise ValueError(f"{name} must be a contiguous 2-D float16 CUDA tensor")
    (two_n, K), M = w16.shape, x.shape[0]
    if x.shape[1] != K or two_n % 2:
        raise ValueError("w16 must be [2N][K] with x [M][K]")
    N = two_n // 2
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    if workspace is None:
        workspace = torch.empty((256,), dtype=torch.uint8, device=x.device)
    _check(lib.zt_q4_gemm_f16w_gate_up_silu(w16.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K,
                                            workspace.data_ptr(), workspace.numel(), _stream_handle(stream)),
           "zt_q4_gemm_f16w_gate_up_silu")
    return y


def lmhead_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.zt_q4_lmhead_workspace_bytes(M, N, K))


def lmhead_argmax(qw, scales, x, logits=None, argmax=None, workspace=None, stream=None):
    """(logits f32 [M][N], argmax int32 [M]); workspace is a uint8 CUDA tensor."""
    torch = _torch()
    M, N, K = _dims(qw, scales, x, 1)
    if logits is None:
        logits = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if argmax is None:
        argmax = torch.empty((M,), dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = torch.empty((lmhead_workspace_bytes(M, N, K),), dtype=torch.uint8, device=x.device)
    _check(lib.zt_q4_lmhead_argmax(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), logits.data_ptr(),
                                   argmax.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                   M, N, K, _stream_handle(stream)), "zt_q4_lmhead_argmax")
    return logits, argmax


def lmhead_argmax_noalloc(qw, scales, x, logits=None, argmax=None, stream=None):
    """lmhead_argmax through the entry point that allocates no device memory
    (its scratch is a static array in the library; see include/zt_q4.h)."""
    torch = _torch()
    M, N, K = _dims(qw, scales, x, 1)
    if logits is None:
        logits = torch.empty((M, N), dtype=torch.float32, device=x.device)
    if argmax is None:
        argmax = torch.empty((M,), dtype=torch.int32, device=x.device)
    _check(lib.zt_q4_lmhead_argmax_noalloc(qw.data_ptr(), scales.data_ptr(), x.data_ptr(), logits.data_ptr(),
                                           argmax.data_ptr(), M, N, K, _stream_handle(stream)),
           "zt_q4_lmhead_argmax_noalloc")
    return logits, argmax


def pass_plan(M: int, K_max: int, n: int = 1) -> Tuple[int, int, int, int, int]:
    """(CTAs per SM, ring stages, k_window, column_blocks, warps per CTA) of
    the decode kernel for these shapes; k_window 0 = activations staged whole;
    column_blocks 2 = the first ceil(M/2) tokens and the rest in separate CTAs
    (no device needed)."""
    c, st, kw, cb, w = _I(0), _I(0), _I(0), _I(0), _I(0)
    _check(lib.zt_q4_pass_plan(M, K_max, n, ctypes.byref(c), ctypes.byref(st), ctypes.byref(kw), ctypes.byref(cb),
                               ctypes.byref(w)), "zt_q4_pass_plan")
    return c.value, st.value, kw.value, cb.value, w.value


class Pass:
    """A decode weight pass: a list of projections run by one persistent kernel.

    Each entry is a dict with torch CUDA tensors: kind ("gemv", "gate_up",
    "lm_head"), qw, scales, x, out (and argmax for "lm_head"), and optional
    wait (read x only after all earlier projections completed).  An optional
    "norm" dict turns on the residual add + RMSNorm prologue (x is then not
    read and may be omitted): residual, gamma, eps, and optionally delta,
    residual_out, x_out.  An optional "rope" dict (gemv only) rotates the
    output's feature pairs: pos (int32 [M] CUDA tensor), head_dim, theta.
    "ld_out" sets the output row stride (default N); "group" the k per scale
    (32, 64 or 128; scales are [rows][K / group]).  The ctypes arrays and
    the workspace are built once; run() only launches."""

    KINDS = {"gemv": ZT_Q4_GEMV, "gate_up": ZT_Q4_GATE_UP_SILU, "lm_head": ZT_Q4_LM_HEAD}

    def __init__(self, projs, workspace=None):
        torch = _torch()
        if not 1 <= len(projs) <= ZT_Q4_PASS_MAX:
            raise ValueError(f"a pass has 1..{ZT_Q4_PASS_MAX} projections")
        self._keep = projs
        arr = (ZtProj * len(projs))()
        self._norms = []
        M = None
        for i, p in enumerate(projs):
            kind = self.KINDS[p["kind"]]
            nm = p.get("norm")
            xs = p.get("x") if nm is None else nm["residual"]
            group = int(p.get("group", 32))
            m, n, k = _dims(p["qw"], p["scales"], xs, 2 if kind == ZT_Q4_GATE_UP_SILU else 1, group)
            if M is None:
                M = m
            elif m != M:
                raise ValueError("all projections of a pass share M")
            am = p.get("argmax")
            norm_ptr = None
            if nm is not None:
                def ptr(key, numel):
                    t = nm.get(key)
                    if t is None:
                        return None
                    if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float16 or t.numel() != numel:
                        raise ValueError(f"norm {key} must be a contiguous CUDA float16 tensor of {numel} elements")
                    return t.data_ptr()
                z = ZtNorm(ptr("residual", m * k), ptr("delta", m * k), ptr("gamma", k),
                           ptr("residual_out", m * k), ptr("x_out", m * k), float(nm.get("eps", 1e-5)))
                self._norms.append(z)
                norm_ptr = ctypes.pointer(z)
            rope_ptr = None
            rp = p.get("rope")
            if rp is not None:
                pos = rp["pos"]
                if not pos.is_cuda or pos.dtype != torch.int32 or pos.numel() != m or not pos.is_contiguous():
                    raise ValueError("rope pos must be a contiguous CUDA int32 tensor with one position per token")
                z = ZtRope(pos.data_ptr(), int(rp["head_dim"]), float(rp.get("theta", 10000.0)))
                self._norms.append(z)
                rope_ptr = ctypes.pointer(z)
            x = p.get("x")
            arr[i] = ZtProj(p["qw"].data_ptr(), p["scales"].data_ptr(), x.data_ptr() if x is not None else None,
                            p["out"].data_ptr(), am.data_ptr() if am is not None else None, kind, n, k,
                            int(bool(p.get("wait", 0))), int(p.get("ld_out", 0)), group, norm_ptr, rope_ptr)
        self.arr, self.n, self.M = arr, len(projs), M
        nbytes = int(lib.zt_q4_pass_workspace_bytes(arr, self.n, M))
        if workspace is None:
            workspace = torch.empty((nbytes,), dtype=torch.uint8, device=projs[0]["out"].device)
        self.workspace = workspace

    def run(self, stream=None):
        _check(lib.zt_q4_pass(self.arr, self.n, self.M, self.workspace.data_ptr(), self.workspace.numel(),
                              _stream_handle(stream)), "zt_q4_pass")

    def run_withholding_phase0(self, stream=None):
        """Error-path test: the pass with CTA 0's phase-0 arrival withheld (see
        zt_q4_pass_test_withhold); the next phase's bounded wait runs out."""
        _check(lib.zt_q4_pass_test_withhold(self.arr, self.n, self.M, self.workspace.data_ptr(),
                                            self.workspace.numel(), _stream_handle(stream)), "zt_q4_pass_test_withhold")

    def run_with_cut_extent(self, rows: int, stream=None):
        """Checked-build test: the pass with every weight extent ``rows`` rows short (see
        zt_q4_pass_test_cut); the copies of the last rows fail their check and are skipped."""
        _check(lib.zt_q4_pass_test_cut(self.arr, self.n, self.M, self.workspace.data_ptr(),
                                       self.workspace.numel(), _stream_handle(stream), rows), "zt_q4_pass_test_cut")

    def errors(self) -> int:
        v = ctypes.c_uint(0)
        _check(lib.zt_q4_pass_errors(self.workspace.data_ptr(), self.n, ctypes.byref(v)), "zt_q4_pass_errors")
        return int(v.value)
