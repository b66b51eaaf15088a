"""Plain float64 CPU oracle for the q4f16 dequantizing GEMV.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library under
``int4_group_quantized_q4f16_b200`` never imports it and shares no code with it.

The arithmetic lives in ``zt_q4_oracle.c`` (plain C, IEEE double, plain loops);
this module only compiles it with gcc and marshals numpy arrays into it.
Each wrapper names the passage the C function follows:

* dequantizing matrix product and f32 LM head -- Zero-TVM forum write-up,
  section "完整的推理流水线" (int4 反量化矩阵乘法; f32 output for the LM head);
* fused gate/up + SiLU -- same write-up, section "内核融合" (fused_ffn.wgsl);
* greedy argmax -- same write-up, section "完整的推理流水线" (贪婪解码采样);
* residual add + RMSNorm -- same write-up, section "内核融合" (add_norm.wgsl),
  read as the standard RMSNorm on the fp16 residual stream;
* rotary position embedding -- same write-up, section "完整的推理流水线" (RoPE
  computed in place in the fused QKV kernel), read as the standard rotation
  of feature pairs (i, i + d/2) within each head.

Format reading (the pages name "q4f16_1" but give no bit layout): group of 32
along K, fp16 scale per group, 8 codes per uint32 low nibble first,
w = (q - 7) * s.  The group size is read from the scales' shape ([rows][K /
group]), so groups of 64 or 128 k use the same functions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "zt_q4_oracle.c")
BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(BUILD_DIR, "libzt_q4_oracle.so")

_P = ctypes.c_void_p
_I = ctypes.c_int


def compile_oracle(source: str = SOURCE, out: str = LIB_PATH) -> str:
    """Compile the oracle C file into a shared library (gcc, -O2, OpenMP).

    ``-ffp-contract=off`` keeps every multiply and add a separately rounded
    IEEE double operation, as written."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _stale(lib: str, source: str) -> bool:
    return (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(source)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _group(K: int, scales: np.ndarray) -> int:
    """Group size from the scales' shape: [rows][K / group]."""
    ng = scales.shape[-1]
    if ng < 1 or K % ng:
        raise ValueError(f"scales with {ng} groups per row do not divide K = {K}")
    return K // ng


def _u16(a) -> np.ndarray:
    """fp16 (or raw uint16 bit patterns) -> contiguous uint16 bit patterns."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError(f"expected float16 or uint16, got {a.dtype}")
    return np.ascontiguousarray(a)


class Oracle:
    """ctypes view of one compiled oracle library (the real one, or a test's
    deliberately broken copy)."""

    def __init__(self, lib_path: Optional[str] = None):
        if lib_path is None:
            if _stale(LIB_PATH, SOURCE):
                compile_oracle()
            lib_path = LIB_PATH
        self.lib_path = lib_path
        lib = ctypes.CDLL(lib_path)
        lib.zto_half_to_double.argtypes = [ctypes.c_uint16]
        lib.zto_half_to_double.restype = ctypes.c_double
        lib.zto_unpack.argtypes = [_P, _I, _I, _P]
        lib.zto_pack.argtypes = [_P, _I, _I, _P]
        lib.zto_gemv.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I]
        lib.zto_gate_up_silu.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I]
        lib.zto_silu.argtypes = [ctypes.c_double]
        lib.zto_silu.restype = ctypes.c_double
        lib.zto_argmax.argtypes = [_P, _I]
        lib.zto_argmax.restype = ctypes.c_int32
        lib.zto_lmhead_argmax.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _P, _I]
        lib.zto_double_to_half.argtypes = [ctypes.c_double]
        lib.zto_double_to_half.restype = ctypes.c_uint16
        lib.zto_add_rmsnorm.argtypes = [_P, _P, _P, _I, _I, ctypes.c_double, _P, _P]
        lib.zto_gemv_rope.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _I, ctypes.c_double, _P, _I]
        lib.zto_dequant_f16.argtypes = [_P, _P, _I, _I, _I, _P]
        lib.zto_gemm_f16w.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I]
        lib.zto_gate_up_silu_f16w.argtypes = [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _I]
        for f in (lib.zto_unpack, lib.zto_pack, lib.zto_gemv,
                  lib.zto_gate_up_silu, lib.zto_lmhead_argmax, lib.zto_add_rmsnorm, lib.zto_gemv_rope,
                  lib.zto_dequant_f16, lib.zto_gemm_f16w, lib.zto_gate_up_silu_f16w):
            f.restype = ctypes.c_int
        self._lib = lib

    # --- format -----------------------------------------------------------
    def half_to_double(self, h) -> np.ndarray:
        h = _u16(h)
        f = self._lib.zto_half_to_double
        return np.array([f(int(v)) for v in h.ravel()], dtype=np.float64).reshape(h.shape)

    def double_to_half(self, v) -> np.ndarray:
        """double -> fp16 bit patterns (uint16), round to nearest even."""
        v = np.asarray(v, dtype=np.float64)
        f = self._lib.zto_double_to_half
        return np.array([f(float(a)) for a in v.ravel()], dtype=np.uint16).reshape(v.shape)

    def unpack(self, qw: np.ndarray, K: int) -> np.ndarray:
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        N = qw.shape[0]
        q = np.empty((N, K), dtype=np.uint8)
        rc = self._lib.zto_unpack(_ptr(qw), N, K, _ptr(q))
        if rc:
            raise ValueError("zto_unpack rejected its arguments")
        return q

    def pack(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.uint8)
        N, K = q.shape
        qw = np.empty((N, K // 8), dtype=np.uint32)
        rc = self._lib.zto_pack(_ptr(q), N, K, _ptr(qw))
        if rc:
            raise ValueError("zto_pack rejected its arguments")
        return qw

    # --- the hot path, in double -------------------------------------------
    @staticmethod
    def _rows(rows):
        if rows is None:
            return None, 0
        r = np.ascontiguousarray(rows, dtype=np.int32)
        return r, int(r.size)

    def gemv(self, qw, scales, x, rows=None, threads: int = 1) -> np.ndarray:
        """y[m][i] = sum_k (q[n_i][k] - 7) * s[n_i][k/32] * x[m][k] in double."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        N, K = qw.shape[0], qw.shape[1] * 8
        M = x.shape[0]
        r, nr = self._rows(rows)
        y = np.empty((M, nr if r is not None else N), dtype=np.float64)
        rc = self._lib.zto_gemv(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s),
                                _ptr(r) if r is not None else None, nr, _ptr(y), threads)
        if rc:
            raise ValueError("zto_gemv rejected its arguments")
        return y

    def dequant_f16(self, qw, scales) -> np.ndarray:
        """w16[n][k] = fp16((q[n][k] - 7) * s[n][k/group]), round to nearest
        even, as binary16 bit patterns viewed as float16 [N][K]."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        N, K = qw.shape[0], qw.shape[1] * 8
        w = np.empty((N, K), dtype=np.uint16)
        if self._lib.zto_dequant_f16(_ptr(qw), _ptr(s), N, K, _group(K, s), _ptr(w)):
            raise ValueError("zto_dequant_f16 rejected its arguments")
        return w.view(np.float16)

    def gemm_f16w(self, qw, scales, x, rows=None, threads: int = 1) -> np.ndarray:
        """y[m][i] = sum_k w16[n_i][k] * x[m][k] in double, w16 as dequant_f16."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        N, K = qw.shape[0], qw.shape[1] * 8
        M = x.shape[0]
        r, nr = self._rows(rows)
        y = np.empty((M, nr if r is not None else N), dtype=np.float64)
        rc = self._lib.zto_gemm_f16w(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s),
                                     _ptr(r) if r is not None else None, nr, _ptr(y), threads)
        if rc:
            raise ValueError("zto_gemm_f16w rejected its arguments")
        return y

    def gate_up_silu_f16w(self, qw, scales, x, rows=None, threads: int = 1) -> np.ndarray:
        """out[m][i] = SiLU(g) * u with g, u the products of the binary16 gate
        and up rows (rows [0,N) gate, [N,2N) up) with x[m], in double."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        N2, K = qw.shape[0], qw.shape[1] * 8
        N, M = N2 // 2, x.shape[0]
        r, nr = self._rows(rows)
        out = np.empty((M, nr if r is not None else N), dtype=np.float64)
        rc = self._lib.zto_gate_up_silu_f16w(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s),
                                             _ptr(r) if r is not None else None, nr, _ptr(out), threads)
        if rc:
            raise ValueError("zto_gate_up_silu_f16w rejected its arguments")
        return out

    def gate_up_silu(self, qw, scales, x, rows=None, threads: int = 1) -> np.ndarray:
        """out[m][i] = SiLU(gate_n . x_m) * (up_n . x_m), rows [0,N) gate, [N,2N) up."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        two_n, K = qw.shape[0], qw.shape[1] * 8
        if two_n % 2:
            raise ValueError("gate/up weight must have an even number of rows")
        N = two_n // 2
        M = x.shape[0]
        r, nr = self._rows(rows)
        out = np.empty((M, nr if r is not None else N), dtype=np.float64)
        rc = self._lib.zto_gate_up_silu(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s),
                                        _ptr(r) if r is not None else None, nr,
                                        _ptr(out), threads)
        if rc:
            raise ValueError("zto_gate_up_silu rejected its arguments")
        return out

    def add_rmsnorm(self, residual, delta, gamma, eps: float):
        """(h, x) as fp16 arrays [M][K]: h = fp16(residual + delta),
        x = fp16(h * gamma / sqrt(mean_k h^2 + eps)); delta may be None."""
        r = _u16(np.atleast_2d(residual))
        M, K = r.shape
        d = _u16(np.atleast_2d(delta)) if delta is not None else None
        if d is not None and d.shape != r.shape:
            raise ValueError("delta must have the residual's shape")
        g = _u16(gamma).ravel()
        if g.size != K:
            raise ValueError("gamma must have K entries")
        h = np.empty((M, K), dtype=np.uint16)
        x = np.empty((M, K), dtype=np.uint16)
        rc = self._lib.zto_add_rmsnorm(_ptr(r), _ptr(d) if d is not None else None, _ptr(g), M, K,
                                       float(eps), _ptr(h), _ptr(x))
        if rc:
            raise ValueError("zto_add_rmsnorm rejected its arguments")
        return h.view(np.float16), x.view(np.float16)

    def gemv_rope(self, qw, scales, x, pos, head_dim: int, theta: float, threads: int = 1) -> np.ndarray:
        """y = W x (double), then feature pairs (i, i + d/2) of every head turned
        by pos[m] * theta^(-2i/d)."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        N, K = qw.shape[0], qw.shape[1] * 8
        M = x.shape[0]
        pos = np.ascontiguousarray(pos, dtype=np.int32).ravel()
        if pos.size != M:
            raise ValueError("one position per token")
        out = np.empty((M, N), dtype=np.float64)
        rc = self._lib.zto_gemv_rope(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s), _ptr(pos), int(head_dim),
                                     float(theta), _ptr(out), threads)
        if rc:
            raise ValueError("zto_gemv_rope rejected its arguments")
        return out

    def silu(self, g: float) -> float:
        return self._lib.zto_silu(float(g))

    def argmax(self, v) -> int:
        v = np.ascontiguousarray(v, dtype=np.float64)
        return int(self._lib.zto_argmax(_ptr(v), int(v.size)))

    def lmhead_argmax(self, qw, scales, x, threads: int = 1):
        """(logits[M][N] in double, argmax[M] int32: lowest index of the max)."""
        qw = np.ascontiguousarray(qw, dtype=np.uint32)
        s = _u16(scales)
        x = _u16(np.atleast_2d(x))
        N, K = qw.shape[0], qw.shape[1] * 8
        M = x.shape[0]
        logits = np.empty((M, N), dtype=np.float64)
        am = np.empty((M,), dtype=np.int32)
        rc = self._lib.zto_lmhead_argmax(_ptr(qw), _ptr(s), _ptr(x), M, N, K, _group(K, s),
                                         _ptr(logits), _ptr(am), threads)
        if rc:
            raise ValueError("zto_lmhead_argmax rejected its arguments")
        return logits, am


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle compiled from this directory's C source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def round_to_half(v: np.ndarray) -> np.ndarray:
    """Round doubles to fp16, round-to-nearest-even (numpy's double->half
    conversion), for comparing against a kernel's single fp16 output rounding."""
    return np.asarray(v, dtype=np.float64).astype(np.float16)
