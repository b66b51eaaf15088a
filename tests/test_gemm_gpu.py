"""GPU parity of the batched (prefill) path: the binary16 dequantization
(bit-exact against the oracle) and the tensor-core GEMM on those weights
(element bound: fp32 accumulation, 2^-14 sum |w16 x|, plus one fp16 ulp)
against the oracle's fp16-weight product (Zero-TVM write-up, limitations
section: batched-prefill shaders, computing in f16)."""
import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import F16_REL_L2, assert_f16_matches, dev, host, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zt():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4


def abs_products_f16w(oracle, qw, scales, x, rows=None):
    """sum_k |w16_nk| |x_mk| by the oracle: |fp16((q - 7) s)| = fp16(|q - 7| |s|),
    i.e. codes 7 + |q - 7| with |s|, against |x|."""
    q = oracle.unpack(qw, qw.shape[1] * 8).astype(np.int16)
    qa = (7 + np.abs(q - 7)).astype(np.uint8)
    sa = np.abs(np.asarray(scales, dtype=np.float16))
    xa = np.abs(np.asarray(x, dtype=np.float16))
    return oracle.gemm_f16w(oracle.pack(qa), sa, xa, rows=rows, threads=8)


def _prefill_x(seed, M, K):
    return np.random.default_rng([seed, 91]).standard_normal((M, K)).astype(np.float16)


@pytest.mark.parametrize("N,K,group", [(1, 32, 32), (3, 96, 32), (256, 3072, 32), (1000, 1024, 64),
                                       (777, 2048, 128), (64, 11008, 32)])
def test_dequant_f16_bit_exact(zt, oracle, N, K, group):
    import torch
    qw, s32, _ = synth.problem(500 + N, N, K, M=1, proj=1)
    s = s32[:, ::group // 32].copy()
    w16 = zt.dequant_f16(dev(qw), dev(s))
    torch.cuda.synchronize()
    assert np.array_equal(host(w16).view(np.uint16), oracle.dequant_f16(qw, s).view(np.uint16))


def test_dequant_f16_edge_scales(zt, oracle):
    """Subnormal, tiny, huge (overflowing to inf), negative and zero scales."""
    import torch
    N, K = 64, 64
    rng = np.random.default_rng(5)
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    bits = np.concatenate([rng.integers(0, 0x0400, 32), rng.integers(0x7800, 0x7C00, 32),
                           rng.integers(0x8000, 0xFC00, 32), [0, 0x8000, 0x3C01, 0x3C03] * 8]).astype(np.uint16)
    s = bits[:N * (K // 32)].reshape(N, K // 32).view(np.float16)
    w16 = zt.dequant_f16(dev(qw), dev(s))
    torch.cuda.synchronize()
    with np.errstate(over="ignore"):
        assert np.array_equal(host(w16).view(np.uint16), oracle.dequant_f16(qw, s).view(np.uint16))


SHAPES = [
    (17, 128, 64),          # one weight tile, one k block, 17 tokens of a 64-token tile
    (1, 200, 96),           # M = 1, ragged N, K % 64 == 32
    (64, 384, 1024),
    (100, 300, 1056),       # ragged everything
    (129, 256, 512),        # just past one 128-token tile
    (256, 1024, 3072),
    (300, 640, 2048),       # 256-token tiles with a ragged second tile
    (40, 3072, 8192),       # Phi-3-mini down projection shape, 40 tokens
    (150, 203, 256),        # tokens as the A operand, N % 8 != 0: element stores
    (200, 360, 128),        # N % 8 == 0 but the last 32 columns ragged: mixed stores
    (128, 1024, 3072),      # exactly one 128-token A tile
]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_gemm_matches_oracle(zt, oracle, M, N, K):
    import torch
    qw, s, _ = synth.problem(600 + M, N, K, M=1, proj=0)
    x = _prefill_x(M + N, M, K)
    ws = torch.empty((zt.gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    y = zt.gemm(dev(qw), dev(s), dev(x), workspace=ws)
    torch.cuda.synchronize()
    assert zt.gemm_errors(ws, N, K) == 0
    ref = oracle.gemm_f16w(qw, s, x, threads=8)
    assert_f16_matches(host(y), ref, f"gemm M{M} N{N} K{K}", abs_products_f16w(oracle, qw, s, x))


@pytest.mark.parametrize("group", [64, 128])
def test_gemm_groups(zt, oracle, group):
    import torch
    M, N, K = 48, 256, 1024
    qw, s32, _ = synth.problem(700 + group, N, K, M=1, proj=2)
    s = s32[:, ::group // 32].copy()
    x = _prefill_x(group, M, K)
    y = zt.gemm(dev(qw), dev(s), dev(x))
    torch.cuda.synchronize()
    assert_f16_matches(host(y), oracle.gemm_f16w(qw, s, x, threads=8), f"gemm group {group}",
                       abs_products_f16w(oracle, qw, s, x))


def test_gemm_full_size_sampled(zt, oracle):
    """Prefill of 512 tokens through the Phi-3-mini qkv projection (3072 ->
    9216) and the LM head rows (3072 -> 32064, fp16 out): sampled rows."""
    import torch
    for N, seed in ((9216, 1), (32064, 2)):
        M, K = 512, 3072
        qw, s, _ = synth.problem(seed, N, K, M=1, proj=0)
        x = _prefill_x(seed, M, K)
        y = host(zt.gemm(dev(qw), dev(s), dev(x)))
        torch.cuda.synchronize()
        rows = np.unique(np.concatenate([[0, 127, 128, N - 1], np.random.default_rng(seed).integers(0, N, 60)]))
        rows = rows.astype(np.int32)
        ref = oracle.gemm_f16w(qw, s, x, rows=rows, threads=8)
        assert_f16_matches(y[:, rows], ref, f"gemm N{N} sampled", abs_products_f16w(oracle, qw, s, x, rows=rows))


def test_gemm_f16w_reuses_dequantized_weights(zt):
    """dequant once + gemm_f16w equals the one-call gemm bit for bit, and
    repeated calls are bit-identical."""
    import torch
    M, N, K = 77, 512, 2048
    qw, s, _ = synth.problem(9, N, K, M=1, proj=3)
    x = dev(_prefill_x(9, M, K))
    qd, sd = dev(qw), dev(s)
    w16 = zt.dequant_f16(qd, sd)
    ws = torch.empty((zt.gemm_f16w_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    a = zt.gemm_f16w(w16, x, workspace=ws)
    b = zt.gemm(qd, sd, x)
    c = zt.gemm(qd, sd, x)
    torch.cuda.synchronize()
    assert zt.gemm_f16w_errors(ws) == 0
    assert np.array_equal(host(a).view(np.uint16), host(b).view(np.uint16))
    assert np.array_equal(host(b).view(np.uint16), host(c).view(np.uint16))


def test_gemm_exact_weights_match_decode_path(zt, oracle):
    """With 7-bit scales the binary16 weights are exact, so the prefill GEMM
    and the decode GEMV compute the same exact products: both within their
    bounds of the exact oracle, for the same 16 tokens."""
    import torch
    M, N, K = 16, 384, 1024
    rng = np.random.default_rng(12)
    qw = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    mant = rng.integers(64, 128, size=(N, K // 32)).astype(np.float64)
    s = (mant * 2.0 ** -13).astype(np.float16)
    x = _prefill_x(12, M, K)
    y_pre = host(zt.gemm(dev(qw), dev(s), dev(x)))
    y_dec = host(zt.gemv(dev(qw), dev(s), dev(x)))
    torch.cuda.synchronize()
    ref = oracle.gemv(qw, s, x, threads=8)
    assert np.array_equal(oracle.gemm_f16w(qw, s, x, threads=8), ref)
    from parity import abs_products
    bound = abs_products(oracle, qw, s, x)
    assert_f16_matches(y_pre, ref, "prefill", bound)
    assert_f16_matches(y_dec, ref, "decode", bound)
    assert rel_l2(y_pre, y_dec) <= F16_REL_L2


@pytest.mark.parametrize("M,N,K", [(1100, 9000, 256), (600, 16000, 96), (2048, 9216, 3072)])
def test_gemm_256_row_tiles_sampled(zt, oracle, M, N, K):
    """Shapes whose grid of 256-row x 256-token tiles covers every SM, so the
    two-accumulator tile runs (ragged N, M and K included); sampled rows on
    both halves of several tiles, every token."""
    import torch
    qw, s, _ = synth.problem(800 + M, N, K, M=1, proj=1)
    x = _prefill_x(M, M, K)
    y = host(zt.gemm(dev(qw), dev(s), dev(x)))
    torch.cuda.synchronize()
    edges = [0, 1, 127, 128, 129, 255, 256, 257, 383, 384, N - 129, N - 128, N - 2, N - 1]
    rows = np.unique(np.concatenate([[r for r in edges if 0 <= r < N],
                                     np.random.default_rng(M).integers(0, N, 40)])).astype(np.int32)
    ref = oracle.gemm_f16w(qw, s, x, rows=rows, threads=8)
    assert_f16_matches(y[:, rows], ref, f"gemm 256-row tiles M{M} N{N} K{K}",
                       abs_products_f16w(oracle, qw, s, x, rows=rows))


@pytest.mark.parametrize("M,N,K", [(512, 3072, 8192), (128, 9216, 8192), (40, 3072, 8192), (200, 1000, 16448)])
def test_gemm_split_k(zt, oracle, M, N, K):
    """Shapes whose tiles cover few SMs run split along K (fp32 partials summed
    in order by a second launch): the Phi-3-mini down projection at 512 and 40
    tokens (weight rows as the A operand at 40), 128 tokens over K = 8192, and
    8 splits with a short last one (K = 16448 = 257 blocks of 64); sampled
    rows, every token; deterministic."""
    import torch
    qw, s, _ = synth.problem(900 + M + N, N, K, M=1, proj=3)
    x = _prefill_x(N, M, K)
    ws = torch.empty((zt.gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    assert ws.numel() > zt.gemm_workspace_bytes(M, N, K) - 1
    qd, sd, xd = dev(qw), dev(s), dev(x)
    y = host(zt.gemm(qd, sd, xd, workspace=ws))
    y2 = host(zt.gemm(qd, sd, xd, workspace=ws))
    torch.cuda.synchronize()
    assert zt.gemm_errors(ws, N, K) == 0
    assert np.array_equal(y.view(np.uint16), y2.view(np.uint16))
    rows = np.unique(np.concatenate([[0, 1, 255, 256, N - 1], np.random.default_rng(M).integers(0, N, 50)]))
    rows = rows.astype(np.int32)
    ref = oracle.gemm_f16w(qw, s, x, rows=rows, threads=8)
    assert_f16_matches(y[:, rows], ref, f"split-K gemm M{M} N{N} K{K}", abs_products_f16w(oracle, qw, s, x, rows=rows))


@pytest.mark.parametrize("M,N,K", [(70, 12288, 256), (128, 12288, 256), (384, 12288, 256), (256, 8192, 4096),
                                   (384, 8192, 4096), (160, 12288, 4096)])
def test_gemm_tile_plans(zt, oracle, M, N, K):
    """Shapes for the remaining tile plans: weight rows as A with a 128-wide
    token tile; 128 x 128 and 128 x 256 token tiles; 256 x 256 split in three
    with 160 tokens in a 256-token tile; sampled rows, every token."""
    import torch
    qw, s, _ = synth.problem(1000 + M, N, K, M=1, proj=2)
    x = _prefill_x(M * 3, M, K)
    ws = torch.empty((zt.gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    y = host(zt.gemm(dev(qw), dev(s), dev(x), workspace=ws))
    torch.cuda.synchronize()
    assert zt.gemm_errors(ws, N, K) == 0
    rows = np.unique(np.concatenate([[0, 63, 64, 127, 128, 255, 256, N - 1],
                                     np.random.default_rng(N).integers(0, N, 40)])).astype(np.int32)
    ref = oracle.gemm_f16w(qw, s, x, rows=rows, threads=8)
    assert_f16_matches(y[:, rows], ref, f"gemm plan M{M} N{N} K{K}", abs_products_f16w(oracle, qw, s, x, rows=rows))


def gate_up_bound_f16w(oracle, qw, s, x, rows):
    """Element bound for SiLU(g) u on binary16 weights, as for the exact
    weights: |SiLU'| <= 1.1, accumulation errors 2^-14 sum |w16 x|."""
    from parity import ACC_BOUND
    N = qw.shape[0] // 2
    g = oracle.gemm_f16w(qw, s, x, rows=rows, threads=8)
    u = oracle.gemm_f16w(qw, s, x, rows=rows + N, threads=8)
    eg = ACC_BOUND * abs_products_f16w(oracle, qw, s, x, rows=rows)
    eu = ACC_BOUND * abs_products_f16w(oracle, qw, s, x, rows=rows + N)
    silu = g / (1.0 + np.exp(-g))
    return (1.1 * eg * np.abs(u) + np.abs(silu) * eu + eg * eu) / ACC_BOUND


@pytest.mark.parametrize("M,N,K,group", [(40, 256, 512, 32), (200, 1000, 1056, 32), (300, 333, 256, 32),
                                         (512, 8192, 3072, 32), (1100, 2048, 1024, 64), (2048, 8192, 3072, 32)])
def test_gemm_gate_up_silu(zt, oracle, M, N, K, group):
    """The fused FFN on the prefill path: gate rows and their up rows in one B
    tile, SiLU(g) u in the epilogue; Phi-3-mini's gate_up (3072 -> 2 x 8192)
    at 512 and 2048 tokens among the shapes; sampled rows, every token."""
    import torch
    qw, s32, _ = synth.problem(1200 + M, 2 * N, K, M=1, proj=2)
    s = s32[:, ::group // 32].copy()
    x = (_prefill_x(M + 7, M, K).astype(np.float32) * 0.5).astype(np.float16)
    ws = torch.empty((zt.gemm_gate_up_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    qd, sd, xd = dev(qw), dev(s), dev(x)
    y = host(zt.gemm_gate_up_silu(qd, sd, xd, workspace=ws))
    w16 = zt.dequant_f16(qd, sd)
    gws = torch.empty((256,), dtype=torch.uint8, device="cuda")
    y2 = host(zt.gemm_f16w_gate_up_silu(w16, xd, workspace=gws))
    torch.cuda.synchronize()
    assert zt.gemm_errors(ws, 2 * N, K) == 0 and zt.gemm_f16w_errors(gws) == 0
    assert np.array_equal(y.view(np.uint16), y2.view(np.uint16))
    rows = np.unique(np.concatenate([[0, 1, 63, 64, 127, 128, N - 1],
                                     np.random.default_rng(N + M).integers(0, N, 40)])).astype(np.int32)
    ref = oracle.gate_up_silu_f16w(qw, s, x, rows=rows, threads=8)
    assert_f16_matches(y[:, rows], ref, f"gate_up M{M} N{N} K{K}", gate_up_bound_f16w(oracle, qw, s, x, rows))
