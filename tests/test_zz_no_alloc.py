"""The allocation-free LM-head entry point (zt_q4_lmhead_argmax_noalloc).

It is for callers that cannot allocate device memory themselves (a plug-in
inside a framework that owns all device allocations, code recorded into a CUDA
graph, a decode loop that must not synchronize on cudaMalloc); its scratch is a
static array inside the library.  Here it is called through the C ABI and
checked against zt_q4_lmhead_argmax with a caller workspace, on two calls in a
row (the second reuses the scratch the first left behind).  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from int4_group_quantized_q4f16_b200 import synth
from parity import assert_f32_matches, check_argmax, dev, host

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice(oracle):
    """Both entry points run the same kernels with the same grid, so logits
    and argmax must agree bit for bit.  The third case (M = 16, the full
    32064-row vocabulary) fills the largest part of the static scratch that
    any legal call uses; it is also checked against the oracle."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from int4_group_quantized_q4f16_b200 import zt_q4
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(1, 32064, 3072, 0), (3, 5000, 1024, 1), (16, 32064, 1024, 2)]   # calls in a row, different shapes
    for M, N, K, seed in cases:
        qw, s, x = synth.problem(seed, N, K, M=M, proj=synth.PROJ_LM_HEAD)
        qw_d, s_d, x_d = dev(qw), dev(s), dev(x)
        ref_logits, ref_am = zt_q4.lmhead_argmax(qw_d, s_d, x_d)
        logits = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        am = torch.full((M,), -1, dtype=torch.int32, device="cuda")
        rc = zt_q4.lib.zt_q4_lmhead_argmax_noalloc(
            ctypes.c_void_p(qw_d.data_ptr()), ctypes.c_void_p(s_d.data_ptr()), ctypes.c_void_p(x_d.data_ptr()),
            ctypes.c_void_p(logits.data_ptr()), ctypes.c_void_p(am.data_ptr()), M, N, K, ctypes.c_void_p(stream))
        assert rc == 0, zt_q4.strerror(rc)
        torch.cuda.synchronize()
        got, want = host(logits), host(ref_logits)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), f"M{M} N{N}: logits differ"
        assert np.array_equal(host(am), host(ref_am)), (host(am), host(ref_am))
        if M == 16:
            ref, _ = oracle.lmhead_argmax(qw, s, x, threads=16)
            assert_f32_matches(got, ref, "noalloc M16")
            check_argmax(host(am), ref)
