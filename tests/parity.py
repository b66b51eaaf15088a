"""Helpers for the GPU parity tests: move seeded inputs to the device, call the
library through its binding, and compare with the oracle.

Tolerances (the stated bar): fp16 outputs relative L2 error <= 1e-3, f32
logits <= 1e-5, argmax exact unless the oracle's top-2 logits are within 1e-3.

On top of that, every element is checked against a bound of one ulp of the
final fp16 rounding plus 2^-14 * sum_k |w_k x_k| (sum_k |w_k x_k| from the
oracle itself: codes 7 + |q - 7| against |x|).  What the bound stands for:
the decode kernel's products are exact, each group of 32 is summed by the
tensor core in fp32 with the zero-point term -7 X_g as its C operand, and the
K / 32 scaled group sums are accumulated in fp32 (one rounding each).  A
worst-case analysis gives about (K / 32 + 2) * 2^-24 times the magnitude of
those intermediates, which run up to ~3.6x sum |w x| (sum (q + 7) s |x|
against sum |q - 7| s |x| for uniform codes): below 2^-14 sum |w x| up to
K ~ 8192, above it for longer rows.  So for K > 8192 the element check is
tighter than the worst case and relies on the rounding errors of random
inputs not lining up (they grow like sqrt(K / 32), far below the bound); the
stated bar remains the relative L2 error.
"""
from __future__ import annotations

import numpy as np

F16_REL_L2 = 1e-3
F32_REL_L2 = 1e-5
ARGMAX_GAP = 1e-3


def dev(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    return torch.from_numpy(a).cuda()


def host(t) -> np.ndarray:
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.int32:
        return t.numpy()
    return t.numpy()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)


ACC_BOUND = 2.0 ** -14


def abs_products(oracle, qw, scales, x, rows=None) -> np.ndarray:
    """sum_k |w_nk| |x_mk| in double, by the oracle: codes 7 + |q - 7| and |x|."""
    q = oracle.unpack(qw, qw.shape[1] * 8).astype(np.int16)
    qa = (7 + np.abs(q - 7)).astype(np.uint8)
    xa = np.abs(np.asarray(x, dtype=np.float16))
    return oracle.gemv(oracle.pack(qa), scales, xa, rows=rows, threads=8)


def gate_up_bound(oracle, qw, s, x, rows):
    """Element bound for SiLU(g) u: with |dg| <= eg, |du| <= eu (accumulation
    errors as for a plain projection) the product moves by at most
    |SiLU'| eg |u| + |SiLU(g)| eu + eg eu, and |SiLU'| <= 1.1."""
    N = qw.shape[0] // 2
    g = oracle.gemv(qw, s, x, rows=rows, threads=8)
    u = oracle.gemv(qw, s, x, rows=rows + N, threads=8)
    eg = ACC_BOUND * abs_products(oracle, qw, s, x, rows=rows)
    eu = ACC_BOUND * abs_products(oracle, qw, s, x, rows=rows + N)
    silu = g / (1.0 + np.exp(-g))
    return (1.1 * eg * np.abs(u) + np.abs(silu) * eu + eg * eu) / ACC_BOUND


def assert_f16_matches(got: np.ndarray, ref: np.ndarray, what: str = "", absprod=None):
    got = np.asarray(got, dtype=np.float16)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite fp16 output"
    r = rel_l2(got, ref)
    assert r <= F16_REL_L2, f"{what}: rel L2 {r:.3e} > {F16_REL_L2}"
    ref16 = ref.astype(np.float16)
    ulp = np.spacing(np.abs(ref16)).astype(np.float64)
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    bound = ulp + (ACC_BOUND * np.asarray(absprod, dtype=np.float64) if absprod is not None else 0.0)
    bad = err > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} outputs outside the element bound, e.g. {list(i)}: "
                             f"got {float(got[i])!r}, exact {float(ref[i])!r}, bound {float(bound[i]):.3g}")


def assert_f32_matches(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape
    r = rel_l2(got, ref)
    assert r <= F32_REL_L2, f"{what}: rel L2 {r:.3e} > {F32_REL_L2}"
    rms = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms + 1e-30, f"{what}: element error too large"


def check_argmax(am_gpu: np.ndarray, logits_ref: np.ndarray, exact_dups=None):
    """argmax exact, unless the oracle's top-2 are within ARGMAX_GAP: then the
    GPU's index must be one of the near-maximal ones.  `exact_dups[m]` lists
    rows known to be exact copies of the top row: then the lowest one must win."""
    for m in range(logits_ref.shape[0]):
        row = logits_ref[m]
        best = int(np.argmax(row))              # numpy: first occurrence = lowest index
        top = row[best]
        near = np.flatnonzero(row >= top - ARGMAX_GAP)
        if exact_dups is not None and exact_dups[m]:
            assert int(am_gpu[m]) == best, f"row {m}: exact duplicate tie must give lowest index {best}"
        elif len(near) == 1:
            assert int(am_gpu[m]) == best, f"row {m}: argmax {am_gpu[m]} != {best}"
        else:
            assert int(am_gpu[m]) in set(near.tolist()), f"row {m}: {am_gpu[m]} not near-max"
