"""Parity at the benchmark's full size and launch configuration: the
Phi-3-mini decode weight pass (32 layers of qkv 3072->9216, o 3072->3072,
gate_up 3072->2x8192 + SiLU*up, down 8192->3072, then the LM head
3072->32064 with f32 logits and argmax; Zero-TVM write-up, sections
"完整的推理流水线" and "内核融合") as one zt_q4_pass call over all 129
projections, built by the same code the benchmark times -- and the same for
the Llama-7B pass (32 layers of qkv 4096->12288, o 4096->4096, gate_up
4096->2x11008 + SiLU*up, down 11008->4096, LM head 4096->32000; the wgpu-llm
page's performance table runs Llama-7B at 4 bits).

The oracle computes sampled rows of every projection of three layers one by
one, and the whole LM head; a second run must reproduce the first bit for
bit.  The chained form (every projection waiting for the previous ones) is
checked the same way, and the same weights with 8 and 16 tokens per
projection (the benchmark's batched decode)."""
import argparse

import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import abs_products, assert_f16_matches, assert_f32_matches, check_argmax, gate_up_bound, host

pytestmark = pytest.mark.gpu

CHECKED_LAYERS = (0, 13, 31)


def _sample_rows(n, seed):
    g = np.random.default_rng([seed, 5])
    return np.unique(np.concatenate([[0, 1, n // 2, n - 2, n - 1], g.integers(0, n, 48)])).astype(np.int64)


@pytest.fixture(scope="module", params=["phi3", "llama7b"])
def full_pass(request):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bench
    from int4_group_quantized_q4f16_b200 import zt_q4
    args = argparse.Namespace(layers=32, seed=0)
    calls, _, _ = bench.build_pass(args, torch.device("cuda", 0), request.param)

    def make(chained):
        projs = []
        for i, d in enumerate(calls):
            e = {"kind": d["p"].kind, "qw": d["qw"], "scales": d["s"], "x": d["x"], "out": d["y"],
                 "wait": 1 if (chained and i) else 0}
            if d["p"].kind == "lm_head":
                e["argmax"] = d["am"]
            projs.append(e)
        return zt_q4.Pass(projs)

    zpass = make(False)
    zpass.run()
    torch.cuda.synchronize()
    assert zpass.errors() == 0
    first = _outputs(calls)
    yield calls, zpass, make, first
    del zpass
    torch.cuda.empty_cache()


def test_full_pass_projection_count(full_pass):
    calls = full_pass[0]
    assert len(calls) == 129
    assert [d["p"].kind for d in calls[:4]] == ["gemv", "gemv", "gate_up", "gemv"]
    assert calls[-1]["p"].kind == "lm_head" and calls[-1]["p"].n_out in (32064, 32000)
    assert {d["p"].K for d in calls} in ({3072, 8192}, {4096, 11008})


def _check_sampled(oracle, calls, outs, layer, what):
    for i, d in enumerate(calls):
        p = d["p"]
        if d["layer"] != layer or p.kind == "lm_head":
            continue
        qw, s, x = synth.proj_inputs(0, layer, p)
        got = outs[i][0]
        rows = _sample_rows(p.n_out, 100 * layer + p.proj_id)
        if p.kind == "gemv":
            ref = oracle.gemv(qw, s, x, rows=rows.astype(np.int32), threads=8)
            bound = abs_products(oracle, qw[rows], s[rows], x)
        else:
            ref = oracle.gate_up_silu(qw, s, x, rows=rows.astype(np.int32), threads=8)
            sub = np.concatenate([rows, rows + p.n_out])
            bound = gate_up_bound(oracle, qw[sub], s[sub], x, np.arange(len(rows), dtype=np.int32))
        assert_f16_matches(got[:, rows], ref, f"{what} layer {layer} {p.name}", bound)


def _check_lm_head(oracle, calls, outs, what):
    d = calls[-1]
    qw, s, x = synth.proj_inputs(0, d["layer"], d["p"])
    logits, am = outs[-1]
    ref, _ = oracle.lmhead_argmax(qw, s, x, threads=8)
    assert_f32_matches(logits, ref, f"{what} lm head")
    check_argmax(am, ref)


def _outputs(calls):
    return [(host(d["y"]).copy(), host(d["am"]).copy() if "am" in d else None) for d in calls]


def _assert_same(a, b, calls):
    for (y0, a0), (y1, a1), d in zip(a, b, calls):
        assert np.array_equal(y0.view(np.uint8), y1.view(np.uint8)), d["p"].name
        if a0 is not None:
            assert np.array_equal(a0, a1)


@pytest.mark.parametrize("layer", CHECKED_LAYERS)
def test_full_pass_sampled_rows(full_pass, oracle, layer):
    calls, _, _, first = full_pass
    _check_sampled(oracle, calls, first, layer, "pass")


def test_full_pass_lm_head(full_pass, oracle):
    calls, _, _, first = full_pass
    _check_lm_head(oracle, calls, first, "pass")


def test_full_pass_repeat_bit_identical(full_pass):
    import torch
    calls, zpass, _, first = full_pass
    zpass.run()
    torch.cuda.synchronize()
    _assert_same(first, _outputs(calls), calls)


def test_full_pass_chained(full_pass, oracle):
    """The chained form (129 phases, a cooperative launch) the benchmark times
    beside the pass.  Its CTA shares differ from the independent form's, and
    with them the K-split of some segments and so the fp32 summation order:
    its outputs are checked against the oracle, and two runs of it against
    each other bit for bit."""
    import torch
    calls, _, make, _ = full_pass
    zchain = make(True)
    zchain.run()
    torch.cuda.synchronize()
    assert zchain.errors() == 0
    one = _outputs(calls)
    zchain.run()
    torch.cuda.synchronize()
    assert zchain.errors() == 0
    _assert_same(one, _outputs(calls), calls)
    for layer in CHECKED_LAYERS:
        _check_sampled(oracle, calls, one, layer, "chained")
    _check_lm_head(oracle, calls, one, "chained")


@pytest.mark.parametrize("M", [8, 16])
def test_full_pass_batched(full_pass, oracle, M):
    """The same 129 projections with M tokens each, as the benchmark's batched
    decode runs them: at M = 8 one 16-warp CTA per SM with 2-deep rings and
    the least partial buffer (Phi-3) or K windows (Llama-7B's 11008-k down
    projection), at M = 16 two column blocks of 8 tokens.  Sampled rows of
    layers 0 and 31, the whole LM head and its argmax."""
    import torch
    from int4_group_quantized_q4f16_b200 import zt_q4
    calls = full_pass[0]
    rng = np.random.default_rng([M, 77])
    projs, xs = [], []
    for d in calls:
        p = d["p"]
        x = rng.standard_normal((M, p.K)).astype(np.float16)
        xs.append(x)
        e = {"kind": p.kind, "qw": d["qw"], "scales": d["s"], "x": torch.from_numpy(x).cuda(),
             "out": torch.empty((M, p.n_out), dtype=torch.float32 if p.kind == "lm_head" else torch.float16,
                                device="cuda")}
        if p.kind == "lm_head":
            e["argmax"] = torch.empty((M,), dtype=torch.int32, device="cuda")
        projs.append(e)
    zp = zt_q4.Pass(projs)
    zp.run()
    torch.cuda.synchronize()
    assert zp.errors() == 0
    for i, d in enumerate(calls):
        p = d["p"]
        if d["layer"] not in (0, 31) or p.kind == "lm_head":
            continue
        qw, s, _ = synth.proj_inputs(0, d["layer"], p)
        x = xs[i]
        rows = _sample_rows(p.n_out, 7 * i + M)
        got = host(projs[i]["out"])
        if p.kind == "gemv":
            ref = oracle.gemv(qw, s, x, rows=rows.astype(np.int32), threads=8)
            bound = abs_products(oracle, qw[rows], s[rows], x)
        else:
            ref = oracle.gate_up_silu(qw, s, x, rows=rows.astype(np.int32), threads=8)
            sub = np.concatenate([rows, rows + p.n_out])
            bound = gate_up_bound(oracle, qw[sub], s[sub], x, np.arange(len(rows), dtype=np.int32))
        assert_f16_matches(got[:, rows], ref, f"M{M} layer {d['layer']} {p.name}", bound)
    d = calls[-1]
    qw, s, _ = synth.proj_inputs(0, d["layer"], d["p"])
    ref, _ = oracle.lmhead_argmax(qw, s, xs[-1], threads=8)
    assert_f32_matches(host(projs[-1]["out"]), ref, f"M{M} lm head")
    check_argmax(host(projs[-1]["argmax"]), ref)
