"""GPU parity of the decode kernel at small batch (M = 2..16) on full-size
shapes, of its K-windowed staging and of its column split: activations that
do not fit in shared memory whole (M x K x 2 bytes beyond ~190 KiB) are
staged in K windows (Llama-7B's down projection 11008 -> 4096 at M = 8), and
more than 8 tokens that would need windows run as two CTAs per row share,
the first ceil(M/2) tokens and the rest (Phi-3 down 8192 -> 3072 at M = 12
and 16: each block whole; Llama-7B down at M = 16: each block in windows)
(Zero-TVM write-up,
sections "完整的推理流水线" and "内核融合": the int4 dequantizing products of
the decoder layer and the fused FFN, here with several tokens per call).

Every output of the full-size calls is compared with the float64 oracle, so
each CTA's first and last tile is covered whatever the grid; larger cases
check densely sampled rows.  zt_q4_pass_plan confirms the path each case
takes."""
import os

import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import (F16_REL_L2, abs_products, assert_f16_matches, assert_f32_matches, check_argmax, dev,
                    gate_up_bound, host, rel_l2)

pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else 8))
EPS = 1e-5


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def _dense_rows(n, seed, every=7):
    g = np.random.default_rng([seed, 11])
    return np.unique(np.concatenate([np.arange(0, n, every), [0, 1, n - 2, n - 1],
                                     g.integers(0, n, 64)])).astype(np.int32)


def _windowed(zt, M, K, n=1):
    return zt.pass_plan(M, K, n)[2] > 0


def _split(zt, M, K, n=1):
    return zt.pass_plan(M, K, n)[3] == 2


# ---------------------------------------------- config 3: gate_up at M > 1 --
@pytest.mark.parametrize("M", [2, 4, 8, 16])
def test_gate_up_full_size_small_batch(zt, oracle, M):
    """gate_up 3072 -> 2 x 8192 with SiLU(g) u at M tokens: every output."""
    N, K = 8192, 3072
    qw, s, x = synth.problem(300 + M, 2 * N, K, M=M, proj=synth.PROJ_GATE_UP)
    got = host(zt.gate_up_silu(dev(qw), dev(s), dev(x)))
    rows = np.arange(N, dtype=np.int32)
    ref = oracle.gate_up_silu(qw, s, x, rows=rows, threads=THREADS)
    assert_f16_matches(got, ref, f"gate_up M{M}", gate_up_bound(oracle, qw, s, x, rows))


# ------------------------------------- down projections past whole-K staging --
@pytest.mark.parametrize("M,N,K,win,split", [(12, 3072, 8192, False, True), (16, 3072, 8192, False, True),
                                             (9, 3072, 8192, False, False), (8, 4096, 11008, True, False),
                                             (16, 4096, 11008, True, True)])
def test_down_full_size_beyond_whole(zt, oracle, M, N, K, win, split):
    """Phi-3 down (8192 -> 3072) at M = 9 (16 columns whole), 12 and 16 (two
    column blocks, each whole) and Llama-7B down (11008 -> 4096) at M = 8 (K
    windows) and 16 (two column blocks of windows): every output."""
    assert (_windowed(zt, M, K), _split(zt, M, K)) == (win, split)
    qw, s, x = synth.problem(400 + M + K, N, K, M=M, proj=synth.PROJ_DOWN)
    got = host(zt.gemv(dev(qw), dev(s), dev(x)))
    ref = oracle.gemv(qw, s, x, threads=THREADS)
    assert_f16_matches(got, ref, f"down M{M} N{N} K{K}", abs_products(oracle, qw, s, x))


def test_down_m4_whole_k(zt, oracle):
    """Llama-7B down at M = 4 still stages x whole (the plan's boundary)."""
    assert not _windowed(zt, 4, 11008)
    qw, s, x = synth.problem(77, 4096, 11008, M=4, proj=synth.PROJ_DOWN)
    got = host(zt.gemv(dev(qw), dev(s), dev(x)))
    assert_f16_matches(got, oracle.gemv(qw, s, x, threads=THREADS), "down M4", abs_products(oracle, qw, s, x))


@pytest.mark.parametrize("M,N,K", [(16, 1000, 16384), (16, 64, 16384), (9, 333, 20000), (5, 96, 40000)])
def test_windowed_ragged(zt, oracle, M, N, K):
    """K = 16384 at M = 16 (the last window ragged), few rows per CTA (K split
    over up to 8 warps inside each window), K not a multiple of 256 (a
    partial last chunk inside the last window; at M = 9 in blocks of 5 + 4
    tokens)."""
    assert _windowed(zt, M, K)
    qw, s, x = synth.problem(500 + N, N, K, M=M, proj=0)
    got = host(zt.gemv(dev(qw), dev(s), dev(x)))
    assert_f16_matches(got, oracle.gemv(qw, s, x, threads=THREADS), f"gemv M{M} N{N} K{K}",
                       abs_products(oracle, qw, s, x))


def test_windowed_many_rounds(zt, oracle):
    """20000 rows at M = 16, K = 11008: several rounds of tiles per CTA, the
    windows staged again in each round (dense sampled rows)."""
    M, N, K = 16, 20000, 11008
    qw, s, x = synth.problem(601, N, K, M=M, proj=1)
    got = host(zt.gemv(dev(qw), dev(s), dev(x)))
    rows = _dense_rows(N, 601)
    ref = oracle.gemv(qw, s, x, rows=rows, threads=THREADS)
    assert_f16_matches(got[:, rows], ref, "many rounds", abs_products(oracle, qw, s, x, rows=rows))


def test_windowed_gate_up(zt, oracle):
    """The fused FFN with K windows (Llama-7B gate_up shape, 2 x 11008 rows, at
    M = 16 with K = 11008: windows and rounds; sampled outputs)."""
    M, N, K = 16, 11008, 11008
    assert _windowed(zt, M, K)
    qw, s, x = synth.problem(602, 2 * N, K, M=M, proj=2)
    got = host(zt.gate_up_silu(dev(qw), dev(s), dev(x)))
    rows = _dense_rows(N, 602, every=13)
    ref = oracle.gate_up_silu(qw, s, x, rows=rows, threads=THREADS)
    assert_f16_matches(got[:, rows], ref, "windowed gate_up", gate_up_bound(oracle, qw, s, x, rows))


@pytest.mark.parametrize("M,N,K", [(16, 6000, 8192), (8, 2500, 11008), (15, 2500, 11008), (9, 3001, 11008)])
def test_windowed_lm_head(zt, oracle, M, N, K):
    """f32 logits and argmax through windows and column blocks (M = 15, 9:
    blocks of 8 + 7 tokens in windows, 5 + 4 whole; the per-CTA maxima of
    both blocks meet in one reduction): every logit, every argmax."""
    assert _windowed(zt, M, K) or _split(zt, M, K)
    qw, s, x = synth.problem(700 + M, N, K, M=M, proj=synth.PROJ_LM_HEAD)
    logits, am = zt.lmhead_argmax(dev(qw), dev(s), dev(x))
    ref, _ = oracle.lmhead_argmax(qw, s, x, threads=THREADS)
    assert_f32_matches(host(logits), ref, f"windowed lm head M{M}")
    check_argmax(host(am), ref)


def test_windowed_single_token(zt, oracle):
    """M = 1 beyond whole-K staging (K = 131072): the single-column kernel's
    windowed path."""
    M, N, K = 1, 200, 131072
    assert _windowed(zt, M, K)
    qw, s, x = synth.problem(801, N, K, M=M, proj=0)
    got = host(zt.gemv(dev(qw), dev(s), dev(x)))
    assert_f16_matches(got, oracle.gemv(qw, s, x, threads=THREADS), "M1 K131072", abs_products(oracle, qw, s, x))


def test_windowed_repeat_bit_identical(zt):
    import torch
    M, N, K = 16, 3000, 11008
    qw, s, x = synth.problem(901, N, K, M=M, proj=0)
    q_d, s_d, x_d = dev(qw), dev(s), dev(x)
    a = host(zt.gemv(q_d, s_d, x_d)).copy()
    b = host(zt.gemv(q_d, s_d, x_d))
    torch.cuda.synchronize()
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


# ------------------------------------- fused prologue / epilogue + windows --
def _norm_inputs(seed, M, K):
    rng = np.random.default_rng([seed, 78])
    res = (rng.standard_normal((M, K)) * 2.0).astype(np.float16)
    dlt = (rng.standard_normal((M, K)) * 0.5).astype(np.float16)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    return res, dlt, gamma


@pytest.mark.parametrize("M,K", [(16, 8192), (15, 11008)])
def test_windowed_norm_prologue(zt, oracle, M, K):
    """Residual add + RMSNorm ahead of a column-split projection (M = 16,
    K = 8192: each block whole; M = 15, K = 11008: each block in windows):
    h bit-exact, x within one fp16 ulp of the oracle, y against the oracle on
    the kernel's own x; a second call is bit-identical."""
    import torch
    N = 1500
    assert _split(zt, M, K)
    qw, s, _ = synth.problem(1001, N, K, M=M, proj=3)
    res, dlt, gamma = _norm_inputs(1001, M, K)
    nm = {"residual": dev(res), "delta": dev(dlt), "gamma": dev(gamma), "eps": EPS}
    nm["residual_out"] = torch.empty_like(nm["residual"])
    nm["x_out"] = torch.empty_like(nm["residual"])
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    p = zt.Pass([{"kind": "gemv", "qw": dev(qw), "scales": dev(s), "out": out, "norm": nm}])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    h_ref, x_ref = oracle.add_rmsnorm(res, dlt, gamma, EPS)
    assert np.array_equal(host(nm["residual_out"]).view(np.uint16), h_ref.view(np.uint16))
    xg = host(nm["x_out"]).copy()
    ulp = np.spacing(np.abs(x_ref)).astype(np.float64)
    assert np.all(np.abs(xg.astype(np.float64) - x_ref.astype(np.float64)) <= ulp)
    got = host(out).copy()
    assert_f16_matches(got, oracle.gemv(qw, s, xg, threads=THREADS), "windowed norm gemv",
                       abs_products(oracle, qw, s, xg))
    assert rel_l2(got, oracle.gemv(qw, s, x_ref, threads=THREADS)) <= F16_REL_L2
    p.run()
    torch.cuda.synchronize()
    assert np.array_equal(got.view(np.uint16), host(out).view(np.uint16))


@pytest.mark.parametrize("M,K", [(16, 8192), (15, 11008)])
def test_windowed_rope_epilogue(zt, oracle, M, K):
    """RoPE on a column-split projection (head_dim 128; each token's own
    position in both blocks), whole and windowed."""
    import torch
    N, d = 1024, 128
    assert _split(zt, M, K)
    qw, s, x = synth.problem(1101, N, K, M=M, proj=0)
    pos = np.random.default_rng(5).integers(0, 4096, M).astype(np.int32)
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    p = zt.Pass([{"kind": "gemv", "qw": dev(qw), "scales": dev(s), "x": dev(x), "out": out,
                  "rope": {"pos": torch.from_numpy(pos).cuda(), "head_dim": d, "theta": 10000.0}}])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    ap = abs_products(oracle, qw, s, x)
    idx = np.arange(N)
    partner = (idx // d) * d + (idx % d + d // 2) % d
    ref = oracle.gemv_rope(qw, s, x, pos, d, 10000.0, threads=THREADS)
    assert_f16_matches(host(out), ref, "windowed rope", ap + ap[:, partner])


# ------------------------------------- a whole layer at M = 16, chained --
def test_windowed_llama_layer_pass_chained(zt, oracle):
    """One Llama-7B-shaped layer at M = 16 as a chained pass (every projection
    waits for the previous ones: a cooperative launch with K windows), plus a
    group-128 projection; sampled rows of every projection, and a second run
    bit-identical."""
    import torch
    M = 16
    layer = synth.llama7b_layer()
    assert _windowed(zt, M, 11008, len(layer) + 1)
    projs, host_in = [], []
    for i, p in enumerate(layer):
        qw, s, x = synth.proj_inputs(3, 0, p, M=M)
        out = torch.empty((M, p.n_out), dtype=torch.float16, device="cuda")
        projs.append({"kind": p.kind, "qw": dev(qw), "scales": dev(s), "x": dev(x), "out": out, "wait": 1 if i else 0})
        host_in.append((p, qw, s, x, 32))
    qw, s, x = synth.problem(1201, 777, 11008, M=M, proj=3)
    s128 = np.ascontiguousarray(s[:, ::4])
    projs.append({"kind": "gemv", "qw": dev(qw), "scales": dev(s128), "x": dev(x), "group": 128, "wait": 1,
                  "out": torch.empty((M, 777), dtype=torch.float16, device="cuda")})
    host_in.append((synth.Proj("g128", "gemv", 11008, 777, 3), qw, s128, x, 128))
    zp = zt.Pass(projs)
    zp.run()
    torch.cuda.synchronize()
    assert zp.errors() == 0
    first = [host(d["out"]).copy() for d in projs]
    for (p, qw, s, x, grp), got in zip(host_in, first):
        rows = _dense_rows(p.n_out, p.proj_id + grp, every=37)
        if p.kind == "gemv":
            ref = oracle.gemv(qw, s, x, rows=rows, threads=THREADS)
            assert_f16_matches(got[:, rows], ref, f"chained {p.name}", abs_products(oracle, qw, s, x, rows=rows))
        else:
            ref = oracle.gate_up_silu(qw, s, x, rows=rows, threads=THREADS)
            assert_f16_matches(got[:, rows], ref, f"chained {p.name}", gate_up_bound(oracle, qw, s, x, rows))
    zp.run()
    torch.cuda.synchronize()
    assert zp.errors() == 0
    for a, d in zip(first, projs):
        assert np.array_equal(a.view(np.uint16), host(d["out"]).view(np.uint16))
