"""The allocation-free linear entry point (nvfp4_linear_noalloc).

It serves callers that cannot allocate device memory -- a plugin inside a
host runtime that owns all device memory, or a serving loop that must stay
out of every allocator -- by keeping its split-K scratch in a fixed array
inside the library.  Its results must match nvfp4_linear (the entry point
that takes a caller-owned workspace) within the GEMM tolerance, on two calls
in a row (the second call reuses the array the first call left behind).

This file is collected last on purpose, so that a failure here does not stop
any other GPU test from running.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import REL_FRO_TOL, cuda, host, rel_fro, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _noalloc(act, g_a, M, wp, g_w, N, K, y, residual=None):
    L = nv.load()
    rc = L.nvfp4_linear_noalloc(act.data_ptr(), g_a.data_ptr(), M, wp.data_ptr(), g_w.data_ptr(), N, K,
                                None if residual is None else residual.data_ptr(), y.data_ptr(), y.stride(0),
                                torch.cuda.current_stream().cuda_stream)
    return rc


@pytest.mark.parametrize("M,N,K", [(16, 4096, 5120), (1, 2048, 2048), (16, 5120, 17408), (3, 200, 320)])
def test_noalloc_matches_workspace_entry_point(M, N, K):
    cuda()
    w = inputs.weight_fp32(120, 1, N, K)
    a = inputs.activation_bf16(120, 2, M, K, 0.01)
    wc, ws, gw = nv.quantize(to_dev(w))
    wp = nv.prepare_weight(wc, ws, N, K)
    act = nv.act_buffer(K)
    _, _, ga = nv.quantize(to_dev(a), act=act)
    ref = host(nv.linear(act, ga, M, wp, gw, N, K))
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = _noalloc(act, ga, M, wp, gw, N, K, y)
        assert rc == 0, nv.load().nvfp4sk_last_error()
        got = host(y)
        assert np.isfinite(got).all(), call
        assert rel_fro(got, ref) <= REL_FRO_TOL, (call, rel_fro(got, ref))
    assert nv.device_status()[0] == 0


def test_noalloc_residual_and_limits():
    cuda()
    M, N, K = 16, 640, 1024
    w = inputs.weight_fp32(121, 1, N, K)
    a = inputs.activation_bf16(121, 2, M, K)
    wc, ws, gw = nv.quantize(to_dev(w))
    wp = nv.prepare_weight(wc, ws, N, K)
    act = nv.act_buffer(K)
    _, _, ga = nv.quantize(to_dev(a), act=act)
    res = to_dev(inputs.bf16_normal(121, 3, (M, N)))
    ref = res.clone()
    nv.linear(act, ga, M, wp, gw, N, K, y=ref, residual=ref)
    out = res.clone()
    assert _noalloc(act, ga, M, wp, gw, N, K, out, residual=out) == 0
    assert rel_fro(host(out), host(ref)) <= REL_FRO_TOL
    # sizes beyond the built-in scratch are refused before anything runs
    L = nv.load()
    big_n = 4096 * 128 + 1
    rc = L.nvfp4_linear_noalloc(act.data_ptr(), ga.data_ptr(), M, wp.data_ptr(), gw.data_ptr(), big_n, K, None,
                                out.data_ptr(), big_n, torch.cuda.current_stream().cuda_stream)
    assert rc == -2 and b"scratch" in L.nvfp4sk_last_error()
    assert L.nvfp4_linear_noalloc_scratch_bytes() <= 4 << 20
