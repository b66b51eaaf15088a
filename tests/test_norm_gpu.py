"""GPU parity of the residual add + RMSNorm prologue of a pass projection
(Zero-TVM write-up, section "内核融合": add_norm.wgsl) against the oracle.

The kernel forms x = fp16(h * r * gamma) in fp32 while the oracle rounds the
double result once, so an x element may sit one fp16 ulp away from the
oracle's; h = fp16(residual + delta) is a single correctly rounded addition
and must match bit for bit.  The projection is then checked against the
oracle evaluated on the kernel's own x (the usual element bound) and against
the oracle's x (relative L2)."""
import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import F16_REL_L2, abs_products, assert_f16_matches, assert_f32_matches, dev, host, rel_l2

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def _norm_inputs(seed, M, K):
    rng = np.random.default_rng([seed, 77])
    res = (rng.standard_normal((M, K)) * 2.0).astype(np.float16)
    dlt = (rng.standard_normal((M, K)) * 0.5).astype(np.float16)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    return res, dlt, gamma


def _check_x(x_gpu, x_ref):
    xg = np.asarray(x_gpu, dtype=np.float16).astype(np.float64)
    xr = np.asarray(x_ref, dtype=np.float16)
    ulp = np.spacing(np.abs(xr)).astype(np.float64)
    assert np.all(np.abs(xg - xr.astype(np.float64)) <= ulp), "normalised x off by more than one fp16 ulp"
    assert rel_l2(xg, xr.astype(np.float64)) <= 1e-3


def _norm_dict(res_d, gamma_d, dlt_d=None, with_outputs=True):
    import torch
    d = {"residual": res_d, "gamma": gamma_d, "eps": EPS}
    if dlt_d is not None:
        d["delta"] = dlt_d
    if with_outputs:
        d["residual_out"] = torch.empty_like(res_d)
        d["x_out"] = torch.empty_like(res_d)
    return d


@pytest.mark.parametrize("kind", ["gemv", "gate_up", "lm_head"])
@pytest.mark.parametrize("M,N,K", [(1, 3072, 3072), (3, 700, 1056), (16, 256, 1024)])
def test_norm_prologue_one_projection(zt, oracle, kind, M, N, K):
    import torch
    rows = 2 * N if kind == "gate_up" else N
    qw, s, _ = synth.problem(900 + M, rows, K, M=M, proj=3)
    res, dlt, gamma = _norm_inputs(M * 1000 + K, M, K)
    nm = _norm_dict(dev(res), dev(gamma), dev(dlt))
    out = torch.empty((M, N), dtype=torch.float32 if kind == "lm_head" else torch.float16, device="cuda")
    proj = {"kind": kind, "qw": dev(qw), "scales": dev(s), "out": out, "norm": nm}
    if kind == "lm_head":
        proj["argmax"] = torch.empty((M,), dtype=torch.int32, device="cuda")
    p = zt.Pass([proj])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    h_ref, x_ref = oracle.add_rmsnorm(res, dlt, gamma, EPS)
    assert np.array_equal(host(nm["residual_out"]).view(np.uint16), h_ref.view(np.uint16))
    x_gpu = host(nm["x_out"])
    _check_x(x_gpu, x_ref)
    got = host(out)
    if kind == "gemv":
        assert_f16_matches(got, oracle.gemv(qw, s, x_gpu, threads=8), "norm gemv", abs_products(oracle, qw, s, x_gpu))
        assert rel_l2(got, oracle.gemv(qw, s, x_ref, threads=8)) <= F16_REL_L2
    elif kind == "gate_up":
        ref = oracle.gate_up_silu(qw, s, x_gpu, threads=8)
        assert rel_l2(got, ref) <= F16_REL_L2
        assert rel_l2(got, oracle.gate_up_silu(qw, s, x_ref, threads=8)) <= F16_REL_L2
    else:
        ref, _ = oracle.lmhead_argmax(qw, s, x_gpu, threads=8)
        assert_f32_matches(got, ref, "norm lm head")


def test_norm_without_delta_and_outputs(zt, oracle):
    """delta NULL (h = residual) and no residual/x outputs: only y is written."""
    import torch
    M, N, K = 2, 512, 2048
    qw, s, _ = synth.problem(31, N, K, M=M, proj=1)
    res, _, gamma = _norm_inputs(5, M, K)
    nm = _norm_dict(dev(res), dev(gamma), None, with_outputs=False)
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    zt.Pass([{"kind": "gemv", "qw": dev(qw), "scales": dev(s), "out": out, "norm": nm}]).run()
    torch.cuda.synchronize()
    h_ref, x_ref = oracle.add_rmsnorm(res, None, gamma, EPS)
    assert np.array_equal(h_ref.view(np.uint16), res.view(np.uint16))
    assert rel_l2(host(out), oracle.gemv(qw, s, x_ref, threads=8)) <= F16_REL_L2


def test_norm_layer_chain(zt, oracle):
    """A decoder-layer-shaped pass: add+norm -> qkv; o projection; add+norm of
    (first norm's h) + (o's output) -> gate_up (waits); down (waits).  Each
    stage is checked on the kernel's actual intermediate values."""
    import torch
    M, H, F = 1, 1024, 2048
    res0, dlt0, g1 = _norm_inputs(1, M, H)
    _, _, g2 = _norm_inputs(2, M, H)
    qkv_w, qkv_s, _ = synth.problem(41, 3 * H, H, M=M, proj=0)
    o_w, o_s, o_x = synth.problem(42, H, H, M=M, proj=1)
    o_s = (o_s.astype(np.float32) * 0.25).astype(np.float16)
    gu_w, gu_s, _ = synth.problem(43, 2 * F, H, M=M, proj=2)
    gu_s = (gu_s.astype(np.float32) * 0.25).astype(np.float16)
    dn_w, dn_s, _ = synth.problem(44, H, F, M=M, proj=3)
    n1 = _norm_dict(dev(res0), dev(g1), dev(dlt0))
    qkv = {"kind": "gemv", "qw": dev(qkv_w), "scales": dev(qkv_s), "norm": n1,
           "out": torch.empty((M, 3 * H), dtype=torch.float16, device="cuda")}
    o = {"kind": "gemv", "qw": dev(o_w), "scales": dev(o_s), "x": dev(o_x),
         "out": torch.empty((M, H), dtype=torch.float16, device="cuda")}
    n2 = _norm_dict(n1["residual_out"], dev(g2), o["out"])
    gu = {"kind": "gate_up", "qw": dev(gu_w), "scales": dev(gu_s), "norm": n2, "wait": 1,
          "out": torch.empty((M, F), dtype=torch.float16, device="cuda")}
    dn = {"kind": "gemv", "qw": dev(dn_w), "scales": dev(dn_s), "x": gu["out"], "wait": 1,
          "out": torch.empty((M, H), dtype=torch.float16, device="cuda")}
    p = zt.Pass([qkv, o, gu, dn])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    h1, x1 = oracle.add_rmsnorm(res0, dlt0, g1, EPS)
    assert np.array_equal(host(n1["residual_out"]).view(np.uint16), h1.view(np.uint16))
    _check_x(host(n1["x_out"]), x1)
    x1g = host(n1["x_out"])
    assert_f16_matches(host(qkv["out"]), oracle.gemv(qkv_w, qkv_s, x1g, threads=8), "qkv",
                       abs_products(oracle, qkv_w, qkv_s, x1g))
    o_out = host(o["out"])
    h2, x2 = oracle.add_rmsnorm(host(n1["residual_out"]), o_out, g2, EPS)
    assert np.array_equal(host(n2["residual_out"]).view(np.uint16), h2.view(np.uint16))
    _check_x(host(n2["x_out"]), x2)
    x2g = host(n2["x_out"])
    assert rel_l2(host(gu["out"]), oracle.gate_up_silu(gu_w, gu_s, x2g, threads=8)) <= F16_REL_L2
    gu_out = host(gu["out"])
    assert_f16_matches(host(dn["out"]), oracle.gemv(dn_w, dn_s, gu_out, threads=8), "down",
                       abs_products(oracle, dn_w, dn_s, gu_out))


def test_norm_deterministic(zt):
    import torch
    M, N, K = 4, 1000, 3072
    qw, s, _ = synth.problem(8, N, K, M=M, proj=0)
    res, dlt, gamma = _norm_inputs(9, M, K)
    nm = _norm_dict(dev(res), dev(gamma), dev(dlt))
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    p = zt.Pass([{"kind": "gemv", "qw": dev(qw), "scales": dev(s), "out": out, "norm": nm}])
    p.run()
    torch.cuda.synchronize()
    first = [host(out).copy(), host(nm["x_out"]).copy()]
    p.run()
    torch.cuda.synchronize()
    assert np.array_equal(first[0].view(np.uint16), host(out).view(np.uint16))
    assert np.array_equal(first[1].view(np.uint16), host(nm["x_out"]).view(np.uint16))
