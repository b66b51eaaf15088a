"""GPU parity of the one-launch decode weight pass (zt_q4_pass) against the
oracle, element by element, on independent and on chained projection lists."""
import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import (abs_products, assert_f16_matches, assert_f32_matches, check_argmax, dev, host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def _proj(kind, N, K, M, seed, proj_id, scale_shift=0):
    import torch
    rows = 2 * N if kind == "gate_up" else N
    qw, s, x = synth.problem(seed, rows, K, M=M, proj=proj_id)
    if scale_shift:
        s = (s.astype(np.float32) * 2.0 ** -scale_shift).astype(np.float16)   # exact: a power of two
    d = {"kind": kind, "qw": dev(qw), "scales": dev(s), "x": dev(x), "host": (qw, s, x), "N": N}
    if kind == "lm_head":
        d["out"] = torch.empty((M, N), dtype=torch.float32, device="cuda")
        d["argmax"] = torch.empty((M,), dtype=torch.int32, device="cuda")
    else:
        d["out"] = torch.empty((M, N), dtype=torch.float16, device="cuda")
    return d


def _check_against_oracle(oracle, d, x_host=None):
    qw, s, x = d["host"]
    if x_host is not None:
        x = x_host
    got = host(d["out"])
    if d["kind"] == "gemv":
        assert_f16_matches(got, oracle.gemv(qw, s, x, threads=8), "pass gemv", abs_products(oracle, qw, s, x))
    elif d["kind"] == "gate_up":
        ref = oracle.gate_up_silu(qw, s, x, threads=8)
        N = d["N"]
        rows = np.arange(N, dtype=np.int32)
        g = oracle.gemv(qw, s, x, rows=rows, threads=8)
        u = oracle.gemv(qw, s, x, rows=rows + N, threads=8)
        eg = 2.0 ** -14 * abs_products(oracle, qw, s, x, rows=rows)
        eu = 2.0 ** -14 * abs_products(oracle, qw, s, x, rows=rows + N)
        silu = g / (1.0 + np.exp(-g))
        bound = (1.1 * eg * np.abs(u) + np.abs(silu) * eu + eg * eu) / 2.0 ** -14
        assert_f16_matches(got, ref, "pass gate_up", bound)
    else:
        ref, _ = oracle.lmhead_argmax(qw, s, x, threads=8)
        assert_f32_matches(got, ref, "pass lm head")
        check_argmax(host(d["argmax"]), ref)


@pytest.mark.parametrize("M", [1, 3, 12])
def test_pass_independent_mixed(zt, oracle, M):
    """qkv/o/gate_up/down-like projections of two layers + an LM head, no waits."""
    import torch
    shapes = [("gemv", 640, 1024), ("gemv", 300, 1024), ("gate_up", 512, 1024), ("gemv", 256, 2048),
              ("gemv", 700, 512), ("gate_up", 96, 256), ("lm_head", 3000, 1024)]
    projs = [_proj(k, N, K, M, 11 + i, i) for i, (k, N, K) in enumerate(shapes)]
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)
    # a second run of the same pass gives identical results
    before = [host(d["out"]).copy() for d in projs]
    p.run()
    torch.cuda.synchronize()
    for b, d in zip(before, projs):
        assert np.array_equal(b.view(np.uint8), host(d["out"]).view(np.uint8))


def test_pass_chained_waits(zt, oracle):
    """x of projection i+1 is the output of projection i (wait set): every
    stage is checked against the oracle on the stage's actual input.  Scales
    are divided by 4 so the chain's activations stay O(1) in fp16."""
    import torch
    M = 2
    dims = [1024, 2048, 512, 1024, 3072, 256]
    projs = []
    for i in range(len(dims) - 1):
        d = _proj("gemv", dims[i + 1], dims[i], M, 40 + i, i, scale_shift=2)
        projs.append(d)
    gu = _proj("gate_up", 1024, dims[-1], M, 60, 9, scale_shift=2)
    projs.append(gu)
    lm = _proj("lm_head", 5000, 1024, M, 61, 10)
    projs.append(lm)
    for i in range(1, len(projs)):
        projs[i]["x"] = projs[i - 1]["out"]
        projs[i]["wait"] = 1
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    _check_against_oracle(oracle, projs[0])
    for i in range(1, len(projs)):
        _check_against_oracle(oracle, projs[i], x_host=host(projs[i - 1]["out"]).astype(np.float16))


def test_pass_matches_single_calls(zt):
    """One projection through the pass equals the single-call entry point bit for bit."""
    import torch
    d = _proj("gemv", 4097, 3072, 1, 5, 0)
    zt.Pass([d]).run()
    single = zt.gemv(d["qw"], d["scales"], d["x"])
    torch.cuda.synchronize()
    assert np.array_equal(host(d["out"]).view(np.uint16), host(single).view(np.uint16))


def test_pass_phases_mixed(zt, oracle):
    """Phases of several independent projections, each later phase reading
    outputs of earlier ones (wait set only on a phase's first projection);
    an LM head in the middle; a ragged K (G % 8 != 0, scales not 16-byte
    aligned rows) whose input is itself an earlier output."""
    import torch
    M = 2
    a = _proj("gemv", 1056, 1024, M, 70, 0, scale_shift=2)        # -> x of c (K = 1056: 33 groups)
    b = _proj("gemv", 768, 1024, M, 71, 1, scale_shift=2)         # -> x of d
    lm = _proj("lm_head", 1000, 1024, M, 72, 2)
    c = _proj("gemv", 2048, 1056, M, 73, 3, scale_shift=2)
    d = _proj("gate_up", 256, 768, M, 74, 4, scale_shift=2)
    e = _proj("gemv", 100, 2048, M, 75, 5, scale_shift=2)
    f = _proj("gemv", 64, 256, M, 76, 6, scale_shift=2)
    c["x"], d["x"], e["x"], f["x"] = a["out"], b["out"], c["out"], d["out"]
    c["wait"] = 1          # phase 1: c, d
    e["wait"] = 1          # phase 2: e, f
    projs = [a, b, lm, c, d, e, f]
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for q in (a, b, lm):
        _check_against_oracle(oracle, q)
    for q, src in ((c, a), (d, b), (e, c), (f, d)):
        _check_against_oracle(oracle, q, x_host=host(src["out"]).astype(np.float16))


def test_pass_many_small_projections(zt, oracle):
    """150 small projections (8..70 outputs, K from one group to a ragged 33
    groups): every CTA's share spans many segments."""
    import torch
    rng = np.random.default_rng(5)
    kinds = ["gemv", "gemv", "gate_up", "gemv"]
    Ks = [32, 96, 288, 1056, 256]
    projs = []
    for i in range(150):
        kind = kinds[i % 4]
        projs.append(_proj(kind, int(rng.integers(8, 71)), Ks[i % 5], 1, 300 + i, i % 5))
    projs[77] = _proj("lm_head", 333, 96, 1, 999, 4)
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)


@pytest.mark.parametrize("M", [2, 5, 8, 9, 16])
def test_pass_batch_sweep(zt, oracle, M):
    """M = 2..16: the single-column kernel is not used, one or two n-tiles."""
    import torch
    shapes = [("gemv", 300, 1024), ("gate_up", 200, 1024), ("lm_head", 777, 512), ("gemv", 64, 3072)]
    projs = [_proj(k, N, K, M, 500 + i, i) for i, (k, N, K) in enumerate(shapes)]
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)


@pytest.mark.parametrize("M", [1, 5, 16])
def test_pass_two_lm_heads(zt, oracle, M):
    """Two LM heads in one list (and one in a later phase): each gets its own
    per-CTA maxima and argmax reduction; a second call starts clean."""
    import torch
    projs = [_proj("lm_head", 4000, 1024, M, 801, 1), _proj("gemv", 640, 1024, M, 802, 2),
             _proj("lm_head", 333, 512, M, 803, 3), _proj("lm_head", 2100, 640, M, 804, 4)]
    projs[3]["x"] = projs[1]["out"]   # reads an earlier output: a second phase
    projs[3]["wait"] = 1
    p = zt.Pass(projs)
    for _ in range(2):   # the counters start from zero again on the second call
        p.run()
        torch.cuda.synchronize()
        assert p.errors() == 0
        for d in projs[:3]:
            _check_against_oracle(oracle, d)
        _check_against_oracle(oracle, projs[3], x_host=host(projs[1]["out"]).astype(np.float16))


@pytest.mark.parametrize("M,K", [(10, 8192), (16, 11008)])
def test_pass_column_split_mixed(zt, oracle, M, K):
    """More than 8 tokens with a long K in the list: every projection runs as
    two column blocks (ceil(M/2) tokens and the rest) sharing each row share, the LM
    head's per-CTA maxima of both blocks meeting in one reduction."""
    import torch
    assert zt.pass_plan(M, K, 5)[3] == 2
    shapes = [("gemv", 300, 1024), ("gate_up", 200, 1024), ("lm_head", 777, 512), ("gemv", 64, K),
              ("lm_head", 1500, K)]
    projs = [_proj(k, N, KK, M, 540 + i, i) for i, (k, N, KK) in enumerate(shapes)]
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)


@pytest.mark.parametrize("N,M,K", [(1, 1, 256), (3, 1, 256), (17, 1, 256), (1, 12, 8192), (3, 16, 11008),
                                   (17, 9, 12288)])
def test_pass_fewer_rows_than_ctas(zt, oracle, N, M, K):
    """A list smaller than the grid: CTAs without rows still write neutral
    LM-head partial maxima (with the column split, for both blocks' tokens)."""
    import torch
    projs = [_proj("gemv", N, K, M, 600 + N, 0), _proj("lm_head", N, K, M, 601 + N, 1)]
    p = zt.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)


def test_pass_bounded_wait_expires_and_reports(zt, oracle):
    """Failure detection without a GPU fault: with CTA 0's phase-0 arrival
    withheld (the test hook), every CTA's bounded wait before phase 1 runs out
    after about 2 s; the kernel sets the error bit, drains its copies and
    returns.  Phase 0's output is still right, and the same pass run normally
    afterwards is clean and correct: the context stayed usable."""
    import time
    import torch
    M = 1
    a = _proj("gemv", 1024, 2048, M, 70, 0)
    b = _proj("gemv", 512, 1024, M, 71, 1, scale_shift=2)
    b["x"] = a["out"]
    b["wait"] = 1
    p = zt.Pass([a, b])
    t0 = time.time()
    p.run_withholding_phase0()
    torch.cuda.synchronize()
    took = time.time() - t0
    assert p.errors() != 0, "the withheld arrival must surface as an expired wait"
    assert took >= 1.5, f"the wait gave up after {took:.2f} s, before its limit"
    _check_against_oracle(oracle, a)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    _check_against_oracle(oracle, a)
    _check_against_oracle(oracle, b, x_host=host(a["out"]).astype(np.float16))
