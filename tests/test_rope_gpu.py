"""GPU parity of the rotary position embedding epilogue of a pass projection
(Zero-TVM write-up, section "完整的推理流水线": RoPE computed in place inside
the fused QKV kernel) against the oracle.

A rotated output mixes the pair's two sums a and b (each within the usual
fp32 accumulation bound 2^-14 sum |w x| of its row), so its element bound is
one fp16 ulp plus 2^-14 times the two rows' sums of |w x|; the angle, sin and
cos are taken in double on both sides."""
import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import ACC_BOUND, F16_REL_L2, abs_products, assert_f16_matches, dev, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def _pair_bound(oracle, qw, s, x, d):
    """per output: 2^-14 (sum |w_n x| + sum |w_partner x|) expressed as the
    absprod argument of assert_f16_matches (which multiplies by 2^-14)."""
    ap = abs_products(oracle, qw, s, x)
    N = ap.shape[1]
    idx = np.arange(N)
    head, j = idx // d, idx % d
    partner = head * d + (j + d // 2) % d
    return ap + ap[:, partner]


def _run_rope(zt, qw, s, x, pos, d, theta, M, N, ld_out=0, out=None):
    import torch
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    proj = {"kind": "gemv", "qw": dev(qw), "scales": dev(s), "x": dev(x), "out": out, "ld_out": ld_out,
            "rope": {"pos": torch.from_numpy(np.asarray(pos, np.int32)).cuda(), "head_dim": d, "theta": theta}}
    p = zt.Pass([proj])
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    return out


@pytest.mark.parametrize("M,N,K,d", [(1, 6144, 3072, 96), (3, 1024, 1024, 128), (16, 192, 256, 64), (2, 96, 1056, 96)])
def test_rope_projection(zt, oracle, M, N, K, d):
    qw, s, x = synth.problem(70 + M, N, K, M=M, proj=0)
    pos = np.random.default_rng(M).integers(0, 4096, M).astype(np.int32)
    pos[0] = 0 if M > 1 else 17
    out = _run_rope(zt, qw, s, x, pos, d, 10000.0, M, N)
    ref = oracle.gemv_rope(qw, s, x, pos, d, 10000.0, threads=8)
    assert_f16_matches(host(out), ref, "rope", _pair_bound(oracle, qw, s, x, d))


def test_rope_large_positions(zt, oracle):
    """Positions up to 2^17: angles of ~10^5 radians, taken in double."""
    M, N, K, d = 4, 384, 512, 96
    qw, s, x = synth.problem(81, N, K, M=M, proj=1)
    pos = np.array([131071, 65536, 12345, 1], np.int32)
    out = _run_rope(zt, qw, s, x, pos, d, 10000.0, M, N)
    ref = oracle.gemv_rope(qw, s, x, pos, d, 10000.0, threads=8)
    assert_f16_matches(host(out), ref, "rope large pos", _pair_bound(oracle, qw, s, x, d))


def test_rope_position_zero_equals_plain(zt):
    """pos = 0 turns nothing: the epilogue returns the plain projection bit for bit."""
    import torch
    M, N, K = 2, 768, 3072
    qw, s, x = synth.problem(82, N, K, M=M, proj=2)
    out = _run_rope(zt, qw, s, x, np.zeros(M, np.int32), 96, 10000.0, M, N)
    plain = torch.empty((M, N), dtype=torch.float16, device="cuda")
    zt.Pass([{"kind": "gemv", "qw": dev(qw), "scales": dev(s), "x": dev(x), "out": plain}]).run()
    torch.cuda.synchronize()
    assert np.array_equal(host(out).view(np.uint16), host(plain).view(np.uint16))


def test_qkv_split_into_one_buffer(zt, oracle):
    """Phi-3-mini QKV: Q and K rows (6144) with RoPE and V rows (3072) plain,
    two projections of one pass writing one [M][9216] buffer through ld_out."""
    import torch
    M, D, K, d = 2, 3072, 3072, 96
    qw, s, x = synth.problem(83, 3 * D, K, M=M, proj=0)
    pos = np.array([7, 300], np.int32)
    out = torch.empty((M, 3 * D), dtype=torch.float16, device="cuda")
    qw_d, s_d, x_d = dev(qw), dev(s), dev(x)
    qk = {"kind": "gemv", "qw": qw_d[:2 * D], "scales": s_d[:2 * D], "x": x_d, "out": out, "ld_out": 3 * D,
          "rope": {"pos": torch.from_numpy(pos).cuda(), "head_dim": d, "theta": 10000.0}}
    v = {"kind": "gemv", "qw": qw_d[2 * D:], "scales": s_d[2 * D:], "x": x_d, "out": out[:, 2 * D:], "ld_out": 3 * D}
    p = zt.Pass([qk, v])
    p.run()
    torch.cuda.synchronize()
    got = host(out)
    ref_qk = oracle.gemv_rope(qw[:2 * D], s[:2 * D], x, pos, d, 10000.0, threads=8)
    assert_f16_matches(got[:, :2 * D], ref_qk, "q/k", _pair_bound(oracle, qw[:2 * D], s[:2 * D], x, d))
    assert_f16_matches(got[:, 2 * D:], oracle.gemv(qw[2 * D:], s[2 * D:], x, threads=8), "v",
                       abs_products(oracle, qw[2 * D:], s[2 * D:], x))


def test_norm_then_rope(zt, oracle):
    """The fused QKV of a layer without its KV append: add + RMSNorm prologue
    and RoPE epilogue on one projection; checked on the kernel's own x."""
    import torch
    M, N, K, d = 1, 1536, 3072, 96
    qw, s, _ = synth.problem(84, N, K, M=M, proj=0)
    rng = np.random.default_rng(9)
    res = rng.standard_normal((M, K)).astype(np.float16)
    dlt = (rng.standard_normal((M, K)) * 0.5).astype(np.float16)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    x_out = torch.empty((M, K), dtype=torch.float16, device="cuda")
    out = torch.empty((M, N), dtype=torch.float16, device="cuda")
    pos = np.array([42], np.int32)
    proj = {"kind": "gemv", "qw": dev(qw), "scales": dev(s), "out": out,
            "norm": {"residual": dev(res), "delta": dev(dlt), "gamma": dev(gamma), "eps": 1e-5, "x_out": x_out},
            "rope": {"pos": torch.from_numpy(pos).cuda(), "head_dim": d, "theta": 10000.0}}
    zt.Pass([proj]).run()
    torch.cuda.synchronize()
    xg = host(x_out)
    ref = oracle.gemv_rope(qw, s, xg, pos, d, 10000.0, threads=8)
    assert_f16_matches(host(out), ref, "norm + rope", _pair_bound(oracle, qw, s, xg, d))
    _, x_ref = oracle.add_rmsnorm(res, dlt, gamma, 1e-5)
    assert rel_l2(host(out), oracle.gemv_rope(qw, s, x_ref, pos, d, 10000.0, threads=8)) <= F16_REL_L2
