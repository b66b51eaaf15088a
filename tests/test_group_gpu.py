"""GPU parity for groups of 64 and 128 k per scale (one fp16 scale shared by 2
or 4 consecutive blocks of 32) in a pass projection.

A group-G projection must equal, bit for bit, the group-32 projection whose
scales repeat each group-G scale G/32 times: the kernel's products and sums
are the same, only the scale loads differ.  It is also checked against the
oracle (which reads the group from the scales' shape)."""
import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import abs_products, assert_f16_matches, assert_f32_matches, check_argmax, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def _run(zt, kind, qw, s, x, N, group):
    import torch
    M = x.shape[0]
    out = torch.empty((M, N), dtype=torch.float32 if kind == "lm_head" else torch.float16, device="cuda")
    proj = {"kind": kind, "qw": dev(qw), "scales": dev(s), "x": dev(x), "out": out, "group": group}
    if kind == "lm_head":
        proj["argmax"] = torch.empty((M,), dtype=torch.int32, device="cuda")
    p = zt.Pass([proj])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    return host(out), (host(proj["argmax"]) if kind == "lm_head" else None)


@pytest.mark.parametrize("group", [64, 128])
@pytest.mark.parametrize("kind,M,N,K", [("gemv", 1, 3072, 3072), ("gemv", 3, 700, 384), ("gate_up", 1, 512, 2048),
                                        ("gate_up", 16, 96, 1024), ("lm_head", 2, 3000, 1024),
                                        ("gemv", 1, 1024, 8192)])
def test_group_matches_repeated_scales_and_oracle(zt, oracle, group, kind, M, N, K):
    if K % group:
        pytest.skip("K must be a multiple of the group")
    rows = 2 * N if kind == "gate_up" else N
    qw, s32, x = synth.problem(1000 + group + M, rows, K, M=M, proj=2)
    sG = s32[:, ::group // 32].copy()                     # one scale per group of G
    s_rep = np.repeat(sG, group // 32, axis=1)            # the same, as group-32 scales
    got, am = _run(zt, kind, qw, sG, x, N, group)
    ref32, am32 = _run(zt, kind, qw, s_rep, x, N, 32)
    assert np.array_equal(got.view(np.uint8), ref32.view(np.uint8)), "group-G differs from repeated group-32 scales"
    if kind == "gemv":
        assert_f16_matches(got, oracle.gemv(qw, sG, x, threads=8), f"group {group}", abs_products(oracle, qw, sG, x))
    elif kind == "gate_up":
        ref = oracle.gate_up_silu(qw, sG, x, threads=8)
        from parity import rel_l2, F16_REL_L2
        assert rel_l2(got, ref) <= F16_REL_L2
    else:
        ref, _ = oracle.lmhead_argmax(qw, sG, x, threads=8)
        assert_f32_matches(got, ref, f"group {group} lm head")
        check_argmax(am, ref)
        assert np.array_equal(am, am32)
