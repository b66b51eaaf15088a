"""The bounds-checked build (libzt_q4_checked.so, -DZT_Q4_CHECKED): on valid
passes no check fires and every output equals the default build's bit for bit;
with the weight extent cut short (zt_q4_pass_test_cut) the checks of the last
rows fire, the copies are skipped, the error bit is set and the context stays
usable.  Nothing here reads outside a buffer: the cut only shrinks the extent
the kernel compares with."""
import importlib.util
import os

import numpy as np
import pytest

from parity import host
from test_pass_gpu import _check_against_oracle, _proj

pytestmark = pytest.mark.gpu


def _load_checked():
    from int4_group_quantized_q4f16_b200 import zt_q4
    path = zt_q4.CHECKED_LIB_PATH
    if not os.path.exists(path):
        from int4_group_quantized_q4f16_b200 import build
        build.build_checked()
    old = os.environ.get("ZT_Q4_LIB")
    os.environ["ZT_Q4_LIB"] = path
    try:
        spec = importlib.util.spec_from_file_location("zt_q4_checked", zt_q4.__file__)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        if old is None:
            del os.environ["ZT_Q4_LIB"]
        else:
            os.environ["ZT_Q4_LIB"] = old
    assert mod.LIB_PATH == path
    return mod


@pytest.fixture(scope="module")
def both():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    return zt_q4, _load_checked()


# K = 1056 (33 groups: scales read directly, a partial last chunk), an LM head, gate_up
SHAPES = [("gemv", 640, 1024), ("gate_up", 512, 1024), ("gemv", 300, 1056), ("gemv", 256, 4096),
          ("lm_head", 3000, 1024)]


def test_build_flags(both):
    zt, zc = both
    assert not zt.is_checked_build() and zc.is_checked_build()
    assert zt.version() == zc.version()


@pytest.mark.parametrize("M", [1, 3, 12])
def test_checked_pass_matches_default(both, oracle, M):
    import torch
    zt, zc = both
    projs = [_proj(k, N, K, M, 71 + i, i) for i, (k, N, K) in enumerate(SHAPES)]
    pd = zt.Pass(projs)
    pd.run()
    torch.cuda.synchronize()
    assert pd.errors() == 0
    want = [host(d["out"]).copy() for d in projs]
    want_am = [host(d["argmax"]).copy() for d in projs if d["kind"] == "lm_head"]
    for d in projs:
        d["out"].fill_(0)
    pc = zc.Pass(projs)
    pc.run()
    torch.cuda.synchronize()
    assert pc.errors() == 0, "a bounds check fired on a valid pass"
    for w, d in zip(want, projs):
        assert np.array_equal(w.view(np.uint8), host(d["out"]).view(np.uint8)), d["kind"]
    assert all(np.array_equal(a, host(d["argmax"])) for a, d in zip(want_am, [d for d in projs if d["kind"] == "lm_head"]))
    for d in projs:
        _check_against_oracle(oracle, d)


def test_checked_single_call_and_chained(both, oracle):
    """One-projection lists (the single-call kernels) and a chained list run clean."""
    import torch
    zt, zc = both
    for M in (1, 4):
        d = _proj("gemv", 1000, 3072, M, 5, 0)
        p = zc.Pass([d])
        p.run()
        torch.cuda.synchronize()
        assert p.errors() == 0
        _check_against_oracle(oracle, d)
    projs = [_proj(k, N, K, 1, 81 + i, i) for i, (k, N, K) in enumerate(SHAPES)]
    for d in projs[1:]:
        d["wait"] = 1
    p = zc.Pass(projs)
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0


@pytest.mark.parametrize("M", [1, 5])
def test_cut_extent_sets_the_error_bit(both, oracle, M):
    import torch
    zt, zc = both
    projs = [_proj(k, N, K, M, 91 + i, i) for i, (k, N, K) in enumerate(SHAPES[:4])]
    p = zc.Pass(projs)
    p.run_with_cut_extent(3)
    torch.cuda.synchronize()
    assert p.errors() & zc.ZT_Q4_ERR_BOUNDS
    # the context is usable and the next (uncut) pass is clean and correct
    p.run()
    torch.cuda.synchronize()
    assert p.errors() == 0
    for d in projs:
        _check_against_oracle(oracle, d)
    # the default build refuses the hook
    pz = zt.Pass(projs)
    assert zt.lib.zt_q4_pass_test_cut(pz.arr, pz.n, pz.M, pz.workspace.data_ptr(), pz.workspace.numel(),
                                      None, 3) == zt.ZT_ERR_UNSUPPORTED
