"""Pins that tie the oracle to something other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with what the format, the mathematics or a library
routine fixes.  ``test_oracle.py`` runs them against the real oracle (all must
pass) and ``test_oracle_mutants.py`` runs them against deliberately broken
copies of it (each copy must fail at least one).

Independent routes used here, none of which calls the oracle's own helpers:

* fp16 decoding -- numpy's float16 -> float64 conversion (library routine);
* nibble order  -- a word's hexadecimal digits read least-significant first
  (string formatting, no shifts or masks);
* sums          -- exact rational arithmetic (``fractions.Fraction``) or
  numpy's float64 matrix product on a dense matrix built by the hex route;
* SiLU          -- closed values: SiLU(0) = 0, SiLU(ln 3) = (3/4) ln 3,
  SiLU(g) - SiLU(-g) = g, SiLU(g) -> g as g -> +inf;
* argmax        -- hand-built logit vectors.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "q4_worked_examples.txt")


# ---------------------------------------------------------------- helpers --
def codes_by_hex(qw: np.ndarray) -> np.ndarray:
    """4-bit codes of packed words, by reading each word's hex digits from the
    least significant end (low nibble first)."""
    qw = np.asarray(qw, dtype=np.uint32)
    N, W = qw.shape
    out = np.empty((N, 8 * W), dtype=np.uint8)
    for n in range(N):
        digits = "".join(format(int(w), "08x")[::-1] for w in qw[n])
        out[n] = [int(c, 16) for c in digits]
    return out


def dense_weights(qw: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """W[n][k] = (q - 7) * s as float64, codes by the hex route."""
    q = codes_by_hex(qw).astype(np.float64)
    s = np.asarray(scales, dtype=np.float16).astype(np.float64)
    return (q - 7.0) * np.repeat(s, 32, axis=1)


def exact_dot(qrow, srow, xrow) -> Fraction:
    """sum_k (q_k - 7) * s_{k//32} * x_k in exact rationals."""
    tot = Fraction(0)
    for k, c in enumerate(qrow):
        tot += (int(c) - 7) * Fraction(float(srow[k // 32])) * Fraction(float(xrow[k]))
    return tot


def small_problem(seed: int, N: int, K: int, M: int = 1):
    g = np.random.default_rng([seed, 12345])
    qw = g.integers(0, 2**32, size=(N, K // 8), dtype=np.uint32)
    s = g.uniform(0.005, 0.02, size=(N, K // 32)).astype(np.float16)
    x = g.standard_normal((M, K)).astype(np.float16)
    return qw, s, x


def parse_golden(path: str = GOLDEN):
    cases, cur = [], None
    with open(path) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "case":
                cur = {"name": tok[1], "kind": tok[2]}
            elif tok[0] == "end":
                cases.append(cur)
                cur = None
            else:
                cur[tok[0]] = tok[1:]
    out = []
    for c in cases:
        K, N, M = int(c["K"][0]), int(c["N"][0]), int(c["M"][0])
        rows = 2 * N if c["kind"] == "gate_up" else N
        d = {
            "name": c["name"], "kind": c["kind"], "K": K, "N": N, "M": M,
            "qw": np.array([int(v, 16) for v in c["qw"]], dtype=np.uint32).reshape(rows, K // 8),
            "scales": np.array([int(v, 16) for v in c["scales"]], dtype=np.uint16)
                        .view(np.float16).reshape(rows, K // 32),
            "x": np.array([int(v, 16) for v in c["x"]], dtype=np.uint16)
                   .view(np.float16).reshape(M, K),
            "y": np.array([float(v) for v in c["y"]], dtype=np.float64).reshape(M, N),
        }
        if "argmax" in c:
            d["argmax"] = np.array([int(v) for v in c["argmax"]], dtype=np.int32)
        out.append(d)
    return out


# ------------------------------------------------------------------- pins --
def pin_half_decode(o):
    """Every one of the 65536 fp16 bit patterns decodes as numpy decodes it."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = o.half_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "NaN patterns decode differently"
    assert np.array_equal(got[~nan], ref[~nan]), "finite/inf fp16 decode mismatch"
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan])), "sign of zero"


def pin_pack_words(o):
    """Hand-written words: codes are stored low nibble first."""
    q = np.array([[1, 2, 3, 4, 5, 6, 7, 8],
                  [15, 0, 0, 0, 0, 0, 0, 0],
                  [0, 0, 0, 0, 0, 0, 0, 15],
                  [0, 1, 2, 3, 4, 5, 6, 7]], dtype=np.uint8)
    want = np.array([[0x87654321], [0x0000000F], [0xF0000000], [0x76543210]], dtype=np.uint32)
    got = o.pack(q)
    assert np.array_equal(got, want), f"pack: {[hex(int(v)) for v in got.ravel()]}"
    assert np.array_equal(o.unpack(want, 8), q), "unpack of hand-written words"


def pin_unpack_matches_hex(o):
    qw, _, _ = small_problem(1, 5, 96)
    assert np.array_equal(o.unpack(qw, 96), codes_by_hex(qw)), "unpack vs hex digits"


def pin_roundtrip(o):
    qw, _, _ = small_problem(2, 7, 256)
    q = o.unpack(qw, 256)
    assert np.array_equal(o.pack(q), qw), "pack(unpack(qw)) != qw"
    g = np.random.default_rng(3)
    q2 = g.integers(0, 16, size=(3, 64), dtype=np.uint8)
    assert np.array_equal(o.unpack(o.pack(q2), 64), q2), "unpack(pack(q)) != q"


def pin_zero_x(o):
    qw, s, x = small_problem(4, 9, 128, M=2)
    y = o.gemv(qw, s, np.zeros_like(x))
    assert np.all(y == 0.0), "zero activations must give exactly zero"


def pin_scale_doubling(o):
    qw, s, x = small_problem(5, 6, 256, M=3)
    s2 = (s.astype(np.float32) * 2).astype(np.float16)          # exact in fp16
    assert np.array_equal(s2.astype(np.float64), 2 * s.astype(np.float64))
    assert np.array_equal(o.gemv(qw, s2, x), 2.0 * o.gemv(qw, s, x)), "y(2s) != 2 y(s)"


def pin_all_ones(o):
    """x = 1: y_n = sum_g s_ng * (sum_{k in g} q_nk - 224), exact."""
    N, K = 16, 256
    qw, s, _ = small_problem(6, N, K)
    x = np.ones((1, K), dtype=np.float16)
    q = codes_by_hex(qw)
    y = o.gemv(qw, s, x)
    for n in range(N):
        want = sum(Fraction(float(s[n, g])) * (int(q[n, 32 * g:32 * g + 32].sum()) - 224)
                   for g in range(K // 32))
        assert Fraction(float(y[0, n])) == want, f"all-ones closed form, row {n}"


def pin_one_hot(o):
    """x = e_k: y_n = (q_nk - 7) * s_n,k/32, exactly, for every k."""
    N, K = 4, 64
    qw, s, _ = small_problem(7, N, K)
    q = codes_by_hex(qw)
    for k in range(K):
        x = np.zeros((1, K), dtype=np.float16)
        x[0, k] = 1.0
        y = o.gemv(qw, s, x)[0]
        want = (q[:, k].astype(np.float64) - 7.0) * s[:, k // 32].astype(np.float64)
        assert np.array_equal(y, want), f"one-hot k={k}"


def pin_brute_force_tiny(o):
    """K = 32, N = 3, M = 2 against exact rationals."""
    qw, s, x = small_problem(8, 3, 32, M=2)
    q = codes_by_hex(qw)
    y = o.gemv(qw, s, x)
    for m in range(2):
        for n in range(3):
            exact = exact_dot(q[n], s[n], x[m])
            mag = sum(abs((int(c) - 7) * float(s[n, k // 32]) * float(x[m, k]))
                      for k, c in enumerate(q[n]))
            assert abs(float(y[m, n]) - float(exact)) <= 1e-14 * mag, f"brute force m={m} n={n}"


def pin_numpy_dense(o):
    """The double matvec against numpy's W @ x^T on a hex-route dense W."""
    qw, s, x = small_problem(9, 64, 512, M=3)
    W = dense_weights(qw, s)
    ref = (W @ x.astype(np.float64).T).T
    y = o.gemv(qw, s, x)
    mag = np.abs(W) @ np.abs(x.astype(np.float64)).T
    assert np.all(np.abs(y - ref) <= 1e-13 * mag.T), "oracle vs numpy dense matvec"


def pin_row_subset(o):
    """A row subset returns exactly the listed rows of the full product."""
    qw, s, x = small_problem(10, 20, 128, M=2)
    full = o.gemv(qw, s, x)
    rows = np.array([19, 0, 7, 7, 3], dtype=np.int32)
    assert np.array_equal(o.gemv(qw, s, x, rows=rows), full[:, rows]), "row subset"


def pin_threads_identical(o):
    qw, s, x = small_problem(11, 33, 256, M=2)
    assert np.array_equal(o.gemv(qw, s, x, threads=1), o.gemv(qw, s, x, threads=4))


def pin_silu_closed_values(o):
    assert o.silu(0.0) == 0.0
    assert math.isclose(o.silu(math.log(3.0)), 0.75 * math.log(3.0), rel_tol=1e-15)
    for g in (0.3, 1.7, 5.0, 11.0):
        assert math.isclose(o.silu(g) - o.silu(-g), g, rel_tol=1e-14), f"odd part at {g}"
    assert o.silu(200.0) == 200.0
    assert abs(o.silu(-200.0)) < 1e-80


def pin_gate_up(o):
    """Gate rows come first: a constant large gate g makes out = g * u."""
    N, K, M = 3, 64, 2
    g = np.random.default_rng(13)
    qw_up = g.integers(0, 2**32, size=(N, K // 8), dtype=np.uint32)
    s_up = g.uniform(0.005, 0.02, size=(N, K // 32)).astype(np.float16)
    qw_gate = np.full((N, K // 8), 0xFFFFFFFF, dtype=np.uint32)   # codes 15 -> w = 8 s
    s_gate = np.full((N, K // 32), 1.0, dtype=np.float16)
    x = np.ones((M, K), dtype=np.float16)
    x[1] = 2.0
    qw = np.concatenate([qw_gate, qw_up])
    s = np.concatenate([s_gate, s_up])
    out = o.gate_up_silu(qw, s, x)
    Wup = dense_weights(qw_up, s_up)
    for m in range(M):
        gate = 8.0 * K * float(x[m, 0])             # 512 or 1024: SiLU(g) == g in double
        u = Wup @ x[m].astype(np.float64)
        assert np.allclose(out[m], gate * u, rtol=1e-13, atol=0), f"gate/up order m={m}"
    # mirrored gate (q -> 14 - q turns g into -g): out(g) - out(-g) = g * u
    qg = g.integers(0, 15, size=(N, K), dtype=np.uint8)
    qw_g = np.array([[sum(int(qg[n, 8 * w + j]) << (4 * j) for j in range(8))
                      for w in range(K // 8)] for n in range(N)], dtype=np.uint32)
    qw_gm = np.array([[sum((14 - int(qg[n, 8 * w + j])) << (4 * j) for j in range(8))
                       for w in range(K // 8)] for n in range(N)], dtype=np.uint32)
    s_g = g.uniform(0.005, 0.02, size=(N, K // 32)).astype(np.float16)
    xr = g.standard_normal((1, K)).astype(np.float16) * np.float16(8)
    a = o.gate_up_silu(np.concatenate([qw_g, qw_up]), np.concatenate([s_g, s_up]), xr)[0]
    b = o.gate_up_silu(np.concatenate([qw_gm, qw_up]), np.concatenate([s_g, s_up]), xr)[0]
    gv = dense_weights(qw_g, s_g) @ xr[0].astype(np.float64)
    uv = Wup @ xr[0].astype(np.float64)
    assert np.allclose(a - b, gv * uv, rtol=1e-12, atol=1e-12), "SiLU odd-part identity"


def pin_argmax(o):
    assert o.argmax([1.0, 3.0, 3.0, 2.0]) == 1, "ties go to the lowest index"
    assert o.argmax([5.0, 5.0]) == 0
    assert o.argmax([float("nan"), -1.0, float("nan")]) == 1, "NaN is -inf"
    assert o.argmax([float("nan"), float("nan")]) == 0, "all NaN -> 0"
    assert o.argmax([-float("inf"), -float("inf"), -3.0]) == 2
    assert o.argmax([0.0, -0.0, 1e-300]) == 2


def pin_lmhead_duplicate_rows(o):
    """An exact duplicate of the top row at a lower index takes the argmax."""
    qw, s, x = small_problem(14, 40, 128, M=2)
    logits, am = o.lmhead_argmax(qw, s, x)
    for m in range(2):
        top = int(np.argmax(logits[m]))
        assert am[m] == top
        qw2, s2 = qw.copy(), s.copy()
        dup = 3 if top != 3 else 5
        lo = min(dup, top)
        qw2[dup], s2[dup] = qw[top], s[top]
        _, am2 = o.lmhead_argmax(qw2, s2, x[m:m + 1])
        assert am2[0] == lo, f"duplicate top row: want {lo}, got {am2[0]}"


def pin_golden(o):
    for c in parse_golden():
        if c["kind"] == "gemv":
            y = o.gemv(c["qw"], c["scales"], c["x"])
            assert np.array_equal(y, c["y"]), f"golden {c['name']}: {y} vs {c['y']}"
        elif c["kind"] == "gate_up":
            y = o.gate_up_silu(c["qw"], c["scales"], c["x"])
            assert np.allclose(y, c["y"], rtol=1e-14, atol=0), f"golden {c['name']}"
        elif c["kind"] == "lm_head":
            logits, am = o.lmhead_argmax(c["qw"], c["scales"], c["x"])
            assert np.array_equal(logits, c["y"]), f"golden {c['name']} logits"
            assert np.array_equal(am, c["argmax"]), f"golden {c['name']} argmax"


# ------------------------------------------------ residual add + RMSNorm ----
# add_norm.wgsl (Zero-TVM write-up, section "内核融合"): the residual add and
# RMSNorm in one step; read as h = fp16(residual + delta),
# x = fp16(h * gamma / sqrt(mean h^2 + eps)).

def _f16(v):
    return np.asarray(v, dtype=np.float64).astype(np.float16)


def pin_double_to_half_is_ieee_round_to_nearest_even(o):
    """Against numpy's double -> binary16 conversion, including exact ties
    (midpoints of adjacent fp16 values), subnormals and the overflow edge."""
    rng = np.random.default_rng(17)
    v = rng.standard_normal(4000) * 10.0 ** rng.integers(-8, 5, 4000)
    a = rng.integers(0, 0x7BFF, 2000, dtype=np.uint16).view(np.float16).astype(np.float64)
    b = (rng.integers(0, 0x7BFF, 2000, dtype=np.uint16) ).view(np.float16).astype(np.float64)
    nxt = np.nextafter(a.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    ties = (a + nxt) / 2.0                        # exact in double
    edge = np.array([0.0, -0.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 65504.0,
                     65519.0, 65520.0, 65536.0, 1e30, -65520.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11])
    vals = np.concatenate([v, -v, ties, -ties, b, edge])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(o.double_to_half(vals), ref)


def pin_rmsnorm_constant_row_gives_gamma(o):
    """A constant row c with eps = 0 normalises to exactly +-1: x = +-gamma
    (gamma varies with k, so a wrong gamma index shows)."""
    K = 64
    gamma = _f16(np.linspace(-3.0, 5.0, K))
    for c in (1.5, -0.375, 96.0):
        h, x = o.add_rmsnorm(_f16(np.full((1, K), c)), None, gamma, 0.0)
        assert np.array_equal(h, _f16(np.full((1, K), c)))
        assert np.array_equal(x[0].astype(np.float64), np.sign(c) * gamma.astype(np.float64))


def pin_rmsnorm_closed_form_ones_and_sevens(o):
    """K = 32: sixteen 1s and sixteen 7s: mean h^2 = (16 + 784) / 32 = 25, so
    with eps = 0 and gamma = 5 the output is h itself.  The row is split as
    residual + delta (both exact in fp16)."""
    h = np.array([1.0] * 16 + [7.0] * 16)
    res = _f16(h - 0.5)
    dlt = _f16(np.full(32, 0.5))
    got_h, x = o.add_rmsnorm(res[None, :], dlt[None, :], _f16(np.full(32, 5.0)), 0.0)
    assert np.array_equal(got_h[0].astype(np.float64), h)
    assert np.array_equal(x[0].astype(np.float64), h)


def pin_rmsnorm_eps_inside_sqrt(o):
    """h = 2^-7 everywhere, eps = 3 * 2^-14: mean h^2 + eps = 2^-12, its root
    2^-6, so x = gamma / 2 exactly."""
    K = 32
    gamma = _f16(np.arange(1, K + 1) * 0.25)
    _, x = o.add_rmsnorm(_f16(np.full((1, K), 2.0 ** -7)), None, gamma, 3 * 2.0 ** -14)
    assert np.array_equal(x[0].astype(np.float64), gamma.astype(np.float64) / 2)


def pin_rmsnorm_scale_invariant(o):
    """eps = 0: scaling the residual by 2^j scales sum h^2 by 4^j and the root
    by 2^j, all exactly, so x does not change."""
    rng = np.random.default_rng(3)
    res = _f16(rng.standard_normal((2, 96)))
    gamma = _f16(rng.uniform(0.5, 2.0, 96))
    _, x0 = o.add_rmsnorm(res, None, gamma, 0.0)
    for j in (-3, 4):
        _, xj = o.add_rmsnorm(_f16(res.astype(np.float64) * 2.0 ** j), None, gamma, 0.0)
        assert np.array_equal(x0.view(np.uint16), xj.view(np.uint16))


def pin_rmsnorm_residual_rounded_to_fp16(o):
    """h is the fp16 sum: 1 + 2^-11 is a tie between 1 and 1 + 2^-10 and goes
    to the even 1; (1 + 2^-10) + 2^-11 goes up to 1 + 2^-9.  delta = -residual
    gives +0 and, with eps > 0, x = 0."""
    K = 32
    res = _f16(np.array([1.0] * 16 + [1.0 + 2.0 ** -10] * 16))
    dlt = _f16(np.full(K, 2.0 ** -11))
    h, _ = o.add_rmsnorm(res[None, :], dlt[None, :], _f16(np.ones(K)), 1e-5)
    assert np.array_equal(h[0].astype(np.float64), np.array([1.0] * 16 + [1.0 + 2.0 ** -9] * 16))
    h, x = o.add_rmsnorm(res[None, :], (-res)[None, :], _f16(np.ones(K)), 1e-5)
    assert np.array_equal(h.view(np.uint16), np.zeros((1, K), dtype=np.uint16))
    assert np.array_equal(x.view(np.uint16), np.zeros((1, K), dtype=np.uint16))


def pin_rmsnorm_rows_independent(o):
    """Each row is normalised by its own mean square: a batch equals its rows
    one at a time, and rows of different scale keep their own result."""
    rng = np.random.default_rng(4)
    res = _f16(rng.standard_normal((3, 64)) * np.array([[0.01], [1.0], [300.0]]))
    dlt = _f16(rng.standard_normal((3, 64)))
    gamma = _f16(rng.uniform(0.5, 2.0, 64))
    h, x = o.add_rmsnorm(res, dlt, gamma, 1e-5)
    for m in range(3):
        hm, xm = o.add_rmsnorm(res[m:m + 1], dlt[m:m + 1], gamma, 1e-5)
        assert np.array_equal(hm.view(np.uint16), h[m:m + 1].view(np.uint16))
        assert np.array_equal(xm.view(np.uint16), x[m:m + 1].view(np.uint16))
    # |x| has unit mean square before gamma: sum (x / gamma)^2 / K ~ 1 in every row
    ms = np.mean((x.astype(np.float64) / gamma.astype(np.float64)) ** 2, axis=1)
    assert np.all(np.abs(ms - 1.0) < 2e-3), ms


# ------------------------------------------------ rotary position embedding ----
# RoPE computed in place in the fused QKV kernel (Zero-TVM write-up, section
# "完整的推理流水线"); read as the standard rotation of pairs (i, i + d/2).

def _rope_problem(seed, M, N, K):
    rng = np.random.default_rng(seed)
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = rng.uniform(0.005, 0.02, size=(N, K // 32)).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    return qw, s, x


def pin_rope_position_zero_is_the_projection(o):
    """pos = 0: cos 0 = 1 and sin 0 = 0 exactly, so every row equals the plain product."""
    qw, s, x = _rope_problem(21, 2, 96, 64)
    got = o.gemv_rope(qw, s, x, np.zeros(2, np.int32), 32, 10000.0)
    assert np.array_equal(got, o.gemv(qw, s, x))


def pin_rope_quarter_turns(o):
    """d = 4, theta = 4 / pi^2: pair 0 (features 0, 2) turns by pos radians and
    pair 1 (features 1, 3) by pos * theta^(-1/2) = pos * pi / 2.  pos = 1
    sends pair 1's (a, b) to (-b, a); pos = 2 to (-a, -b); pos = 4 back."""
    qw, s, x = _rope_problem(22, 1, 8, 64)
    y = o.gemv(qw, s, x)[0]
    theta = 4.0 / np.pi ** 2
    for pos, (ca, cb) in ((1, ((0, -1), (1, 0))), (2, ((-1, 0), (0, -1))), (4, ((1, 0), (0, 1)))):
        got = o.gemv_rope(qw, s, x, np.array([pos], np.int32), 4, theta)[0]
        for h in (0, 4):
            a, b = y[h + 1], y[h + 3]
            assert abs(got[h + 1] - (ca[0] * a + ca[1] * b)) <= 1e-12 * (abs(a) + abs(b))
            assert abs(got[h + 3] - (cb[0] * a + cb[1] * b)) <= 1e-12 * (abs(a) + abs(b))
        # pair 0 turns by pos radians (math library cos / sin of an integer)
        a, b = y[0], y[2]
        c, sn = np.cos(float(pos)), np.sin(float(pos))
        assert abs(got[0] - (a * c - b * sn)) <= 1e-12 * (abs(a) + abs(b))
        assert abs(got[2] - (b * c + a * sn)) <= 1e-12 * (abs(a) + abs(b))


def pin_rope_keeps_pair_lengths(o):
    """A rotation keeps a^2 + b^2 of every pair; the pairing is (i, i + d/2):
    pairing neighbours (2i, 2i + 1) instead breaks this for the true pairs."""
    qw, s, x = _rope_problem(23, 3, 192, 96)
    d = 96
    y = o.gemv(qw, s, x)
    got = o.gemv_rope(qw, s, x, np.array([5, 1000, 31], np.int32), d, 10000.0)
    for h in range(2):
        for i in range(d // 2):
            n, n2 = h * d + i, h * d + i + d // 2
            r0 = y[:, n] ** 2 + y[:, n2] ** 2
            r1 = got[:, n] ** 2 + got[:, n2] ** 2
            assert np.all(np.abs(r1 - r0) <= 1e-12 * r0 + 1e-300)
    assert not np.allclose(got, y)


def pin_rope_frequency_per_pair(o):
    """With theta = 2^8 and d = 16, pair i turns by pos * 2^(-i): for pos =
    2^7 pair 7 turns by exactly 1 radian, pair 0 by 128 -- each token uses its
    own position."""
    qw, s, x = _rope_problem(24, 2, 16, 32)
    y = o.gemv(qw, s, x)
    got = o.gemv_rope(qw, s, x, np.array([128, 0], np.int32), 16, 256.0)
    for i, phi in ((7, 1.0), (0, 128.0), (3, 16.0)):
        a, b = y[0, i], y[0, i + 8]
        assert abs(got[0, i] - (a * np.cos(phi) - b * np.sin(phi))) <= 1e-11 * (abs(a) + abs(b))
        assert abs(got[0, i + 8] - (b * np.cos(phi) + a * np.sin(phi))) <= 1e-11 * (abs(a) + abs(b))
    assert np.array_equal(got[1], y[1])          # the second token sits at position 0


# ------------------------------------------------------- group sizes ----
# q4f16_1 groups 32 k per scale; groups of 64 and 128 (one scale shared by
# 2 or 4 consecutive blocks of 32) are the same formula.

def pin_group_64_and_128_are_repeated_32(o):
    """A group-G scale array equals the group-32 array with every scale
    repeated G / 32 times: the products, the sums and their order are the
    same, so the results are identical bit for bit (gemv, gate/up, LM head)."""
    rng = np.random.default_rng(31)
    K, N, M = 512, 24, 2
    qw = rng.integers(0, 2 ** 32, size=(2 * N, K // 8), dtype=np.uint64).astype(np.uint32)
    x = rng.standard_normal((M, K)).astype(np.float16)
    for G in (64, 128):
        sG = rng.uniform(0.005, 0.02, size=(2 * N, K // G)).astype(np.float16)
        s32 = np.repeat(sG, G // 32, axis=1)
        assert np.array_equal(o.gemv(qw, sG, x), o.gemv(qw, s32, x))
        assert np.array_equal(o.gate_up_silu(qw, sG, x), o.gate_up_silu(qw, s32, x))
        la, aa = o.lmhead_argmax(qw, sG, x)
        lb, ab = o.lmhead_argmax(qw, s32, x)
        assert np.array_equal(la, lb) and np.array_equal(aa, ab)


def pin_group_whole_row_brute_force(o):
    """One scale per row (group = K = 64): y = s * sum_k (q_k - 7) x_k, in
    exact rationals."""
    from fractions import Fraction
    rng = np.random.default_rng(32)
    K, N = 64, 3
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = rng.uniform(0.5, 2.0, size=(N, 1)).astype(np.float16)
    x = rng.standard_normal((1, K)).astype(np.float16)
    q = codes_by_hex(qw)
    y = o.gemv(qw, s, x)
    for n in range(N):
        exact = Fraction(float(s[n, 0])) * sum(Fraction(int(q[n, k]) - 7) * Fraction(float(x[0, k])) for k in range(K))
        assert abs(Fraction(y[0, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)




# -------------------------------------- batched prefill on fp16 weights ----
# The limitations section of the Zero-TVM write-up: batched-prefill shaders
# exist (not wired in), and the shaders compute in f16.  Read as
# w16 = fp16((q - 7) * s), then y = sum_k w16 x in plain k order.

GOLDEN_F16 = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "q4_dequant_f16.txt")


def _golden_f16():
    ws, ys = [], []
    with open(GOLDEN_F16) as fh:
        for raw in fh:
            tok = raw.split("#", 1)[0].split()
            if not tok:
                continue
            if tok[0] == "w":
                ws.append((int(tok[1]), int(tok[2], 16), int(tok[3], 16)))
            elif tok[0] == "y":
                ys.append((int(tok[1]), int(tok[2]), int(tok[3], 16), int(tok[4], 16), float(tok[5])))
    return ws, ys


def _row_of_codes(code: int, K: int) -> np.ndarray:
    word = int("".join([format(code, "x")] * 8), 16)       # eight equal hex digits
    return np.full((1, K // 8), word, dtype=np.uint32)


def pin_dequant_f16_golden(o):
    ws, ys = _golden_f16()
    for code, sbits, wbits in ws:
        qw = _row_of_codes(code, 32)
        s = np.array([[sbits]], dtype=np.uint16).view(np.float16)
        got = o.dequant_f16(qw, s).view(np.uint16)
        assert np.all(got == wbits), f"code {code} scale {sbits:#06x}: {got[0, 0]:#06x} vs {wbits:#06x}"
    for K, code, sbits, xbits, y in ys:
        qw = _row_of_codes(code, K)
        s = np.full((1, K // 32), sbits, dtype=np.uint16).view(np.float16)
        x = np.full((1, K), xbits, dtype=np.uint16).view(np.float16)
        assert o.gemm_f16w(qw, s, x)[0, 0] == y


def pin_dequant_f16_is_numpy_rounding(o):
    """Against numpy's double -> binary16 conversion of the exact product
    (codes by the hex route), over random codes and scales from subnormal to
    large, groups 32 and 64."""
    rng = np.random.default_rng(41)
    N, K = 24, 256
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    q = codes_by_hex(qw).astype(np.float64) - 7.0
    for G in (32, 64):
        sb = rng.integers(0, 0x7C00, size=(N, K // G), dtype=np.uint16)
        s = sb.view(np.float16)
        with np.errstate(over="ignore"):
            ref = (q * np.repeat(s.astype(np.float64), G, axis=1)).astype(np.float16)
        assert np.array_equal(o.dequant_f16(qw, s).view(np.uint16), ref.view(np.uint16))


def pin_gemm_f16w_exact_when_scales_are_short(o):
    """Scales with at most 7 significant bits make (q - 7) s exact in fp16
    (4 + 7 bits), so the fp16-weight product equals the exact one bit for bit."""
    rng = np.random.default_rng(42)
    N, K, M = 16, 192, 3
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    mant = rng.integers(64, 128, size=(N, K // 32)).astype(np.float64)
    s = (mant * 2.0 ** rng.integers(-16, -8, size=(N, K // 32))).astype(np.float16)
    assert np.array_equal(s.astype(np.float64), mant * 2.0 ** np.round(np.log2(s.astype(np.float64) / mant)))
    x = rng.standard_normal((M, K)).astype(np.float16)
    assert np.array_equal(o.gemm_f16w(qw, s, x), o.gemv(qw, s, x))


def pin_gemm_f16w_one_hot_and_brute_force(o):
    """x = e_k picks numpy's fp16 rounding of (q - 7) s at column k; a tiny
    case summed in exact rationals over numpy-rounded weights."""
    rng = np.random.default_rng(43)
    N, K = 5, 64
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = rng.uniform(0.3, 3.0, size=(N, K // 32)).astype(np.float16)
    w16 = ((codes_by_hex(qw).astype(np.float64) - 7.0) * np.repeat(s.astype(np.float64), 32, axis=1)).astype(np.float16)
    eye = np.eye(K, dtype=np.float16)
    y = o.gemm_f16w(qw, s, eye)                       # y[k][n] = w16[n][k]
    assert np.array_equal(y.T, w16.astype(np.float64))
    x = rng.standard_normal((3, K)).astype(np.float16)
    y = o.gemm_f16w(qw, s, x)
    for m in range(3):
        for n in range(N):
            exact = sum(Fraction(float(w16[n, k])) * Fraction(float(x[m, k])) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 2 ** 48) + Fraction(1, 2 ** 200)


def pin_gemm_f16w_rows_and_tokens(o):
    """Row subsets and token rows are independent: a subset and a single token
    return the same numbers as the full product."""
    rng = np.random.default_rng(44)
    N, K, M = 40, 96, 4
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = rng.uniform(0.005, 0.02, size=(N, K // 32)).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    full = o.gemm_f16w(qw, s, x)
    rows = np.array([39, 0, 17, 17, 5], dtype=np.int32)
    assert np.array_equal(o.gemm_f16w(qw, s, x, rows=rows), full[:, rows])
    for m in range(M):
        assert np.array_equal(o.gemm_f16w(qw, s, x[m:m + 1])[0], full[m])


def pin_gate_up_f16w_golden(o):
    with open(GOLDEN_F16) as fh:
        cases = [raw.split("#", 1)[0].split() for raw in fh]
    cases = [c for c in cases if c and c[0] == "f"]
    assert len(cases) == 2
    for _, K, gc, gs, uc, us, xb, out in cases:
        K = int(K)
        qw = np.concatenate([_row_of_codes(int(gc), K), _row_of_codes(int(uc), K)])
        s = np.array([[int(gs, 16)] * (K // 32), [int(us, 16)] * (K // 32)], dtype=np.uint16).view(np.float16)
        x = np.full((1, K), int(xb, 16), dtype=np.uint16).view(np.float16)
        assert o.gate_up_silu_f16w(qw, s, x)[0, 0] == float(out)


def pin_gate_up_f16w_exact_when_scales_are_short(o):
    """7-bit scales make every w16 exact: the fp16-weight fused FFN equals the
    exact one (whose gate/up order and SiLU are pinned above) bit for bit,
    for all rows and for a row subset."""
    rng = np.random.default_rng(45)
    N, K, M = 12, 128, 3
    qw = rng.integers(0, 2 ** 32, size=(2 * N, K // 8), dtype=np.uint64).astype(np.uint32)
    s = (rng.integers(64, 128, size=(2 * N, K // 32)).astype(np.float64) * 2.0 ** -10).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    assert np.array_equal(o.gate_up_silu_f16w(qw, s, x), o.gate_up_silu(qw, s, x))
    rows = np.array([11, 0, 5], dtype=np.int32)
    assert np.array_equal(o.gate_up_silu_f16w(qw, s, x, rows=rows), o.gate_up_silu(qw, s, x)[:, rows])



ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
