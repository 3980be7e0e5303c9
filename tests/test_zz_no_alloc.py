"""The wgrad entry point that allocates nothing (GPU).

fp8_block_gemm_wgrad_static_ws serves callers that cannot hand the library
a device workspace (no memory manager of their own, or a framework
allocator that already holds the GPU's memory): its split-schedule
workspace is an array inside the library.  Called through the C ABI on a
wgrad that the split schedule cuts across CTA pairs, it must give what the
workspace-taking entry point gives, within the parity tests' bound, on two
calls in a row (the second reuses the array the first left behind).

This file is collected last, so that a run which stops at the first failure
has run every other test before it; it passes alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import blockwise_fp8_pretraining_b200 as fp8
import oracle
from blockwise_fp8_pretraining_b200 import synthetic as syn

from _parity import REL_TOL, ABS_TOL, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fp8.load()
    fp8.fp8_clear_error()
    # a small shape, so the split schedule (which uses the workspace) needs
    # its least-work threshold lifted
    fp8.fp8_set_gemm_split_min_work(0)
    yield
    fp8.fp8_set_gemm_split_min_work(fp8.GEMM_SPLIT_MIN_WORK_DEFAULT)
    assert fp8.fp8_get_error() == 0


def test_static_workspace_wgrad_matches_the_workspace_entry_point_twice():
    N, K, M = 1280, 2304, 4096          # 45 tiles of 32 slabs: cut across the CTA pairs
    assert any(kb0 > 0 for _, _, kb0, _, _, _ in fp8.fp8_selftest_gemm_schedule(N, K, M, 74, True))
    d = dev()
    g = syn.generator(4242)
    dy = syn.normal_bf16((M, N), 1e-3, g)
    x = syn.activation_bf16(M, K, K // 100, 30.0, g)
    _, _, dyqT, sdyT = fp8.fp8_quantize_act_1x128(dy.to(d), fp8.COLWISE)
    _, _, xqT, sxT = fp8.fp8_quantize_act_1x128(x.to(d), fp8.COLWISE)
    ref = fp8.fp8_block_gemm_wgrad(dyqT, sdyT, xqT, sxT, workspace=fp8.fp8_gemm_workspace())

    lib = fp8.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    outs = []
    for _ in range(2):
        dw = torch.full((N, K), float("nan"), dtype=torch.bfloat16, device=d)
        st = lib.fp8_block_gemm_wgrad_static_ws(P(dyqT), P(sdyT), P(xqT), P(sxT), P(dw), N, K, M, stream)
        assert st == 0, (st, fp8.fp8_last_cuda_error())
        outs.append(dw)
    torch.cuda.synchronize()
    assert fp8.fp8_get_error() == 0

    # the oracle's bound S on a stratified row sample; the comparison itself
    # is between the two entry points, element by element on those rows
    rows = np.unique(np.concatenate([np.arange(0, N, 97), [N - 1]]))
    dyqT_o, sdyT_o = oracle.quantize_act_colwise(syn.bf16_bits(dy))
    xqT_o, sxT_o = oracle.quantize_act_colwise(syn.bf16_bits(x))
    _, bound = oracle.gemm_wgrad(dyqT_o, sdyT_o, xqT_o, sxT_o, rows=rows)
    r = torch.as_tensor(rows, device=d)
    want = ref[r].float().cpu().numpy().astype(np.float64)
    for i, dw in enumerate(outs):
        got = dw[r].float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"call {i}: output not fully written"
        err = np.abs(got - want)
        assert np.all(err <= REL_TOL * bound + ABS_TOL), f"call {i}: {int((err > REL_TOL * bound + ABS_TOL).sum())} elements"
        assert torch.isfinite(dw.float()).all(), f"call {i}: output not fully written"
