"""GPU: the gate+up linear with SwiGLU and NVFP4 quantisation in its epilogue
(nvfp4_linear_swiglu) against the two-launch sequence it replaces
(nvfp4_linear of the [2F, K] gate+up weight, then nvfp4_swiglu_quantize with
the same static scale): the prepared activations must be byte-identical, on
the verify step's shape and on small shapes, under grids that split tiles
over 1..many CTAs (owner / contributor reductions of both accumulators).
The two-launch sequence is itself gated against the oracle elsewhere (linear
within 1e-3, SwiGLU quantiser bit-exact)."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _operands(M, F, K, seed):
    w = torch.from_numpy(inputs.weight_fp32(70 + seed, 1, 2 * F, K)).cuda()
    codes, scales, g_w = nv.quantize(w)
    w_p = nv.prepare_weight(codes, scales, 2 * F, K)
    a = inputs.activation_bf16(70 + seed, 2, M, K, True).cuda()
    act = nv.act_buffer(K)
    _, _, g_a = nv.quantize(a, act=act)
    return w_p, g_w, act, g_a


def _two_launches(act, g_a, M, w_p, g_w, F, K, g_out):
    gu = nv.linear(act, g_a, M, w_p, g_w, 2 * F, K)
    ref = nv.act_buffer(F)
    out = (None, None, torch.empty(1, dtype=torch.float32, device="cuda"))
    nv.swiglu_quantize(gu, out, act=ref, g_in=g_out)
    return gu, ref


@pytest.mark.parametrize("M,F,K,ctas", [(16, 17408, 5120, 0), (16, 17408, 5120, 37), (1, 17408, 5120, 0),
                                        (5, 256, 512, 0), (16, 384, 1536, 5), (7, 1024, 3072, 3),
                                        (16, 128, 64, 0)])
def test_fused_equals_two_launches(M, F, K, ctas):
    cuda()
    nv.set_option(nv.OPT_LINEAR_CTAS, ctas)
    try:
        w_p, g_w, act, g_a = _operands(M, F, K, F % 7 + M)
        # a realistic static scale: the dynamic one of this very output
        gu = nv.linear(act, g_a, M, w_p, g_w, 2 * F, K)
        _, _, g_dyn = nv.swiglu_quantize(gu, (None, None, torch.empty(1, dtype=torch.float32, device="cuda")),
                                         act=nv.act_buffer(F))
        g_out = g_dyn.clone()
        _, ref = _two_launches(act, g_a, M, w_p, g_w, F, K, g_out)
        fused = nv.act_buffer(F)
        nv.linear_swiglu(act, g_a, M, w_p, g_w, F, K, g_out, fused)
        torch.cuda.synchronize()
        assert nv.device_status() == (0, 0)
        assert torch.equal(fused.cpu(), ref.cpu())
    finally:
        nv.set_option(nv.OPT_LINEAR_CTAS, 0)


def test_fused_repeatable_and_rows_independent():
    """Bit-identical across calls, and the rows of an M = 16 call equal the
    same rows computed alone (no row leaks into another)."""
    cuda()
    M, F, K = 16, 2048, 5120
    w_p, g_w, act16, g_a = _operands(M, F, K, 3)
    g_out = torch.full((1,), 0.01, dtype=torch.float32, device="cuda")
    a = nv.act_buffer(F)
    b = nv.act_buffer(F)
    nv.linear_swiglu(act16, g_a, M, w_p, g_w, F, K, g_out, a)
    nv.linear_swiglu(act16, g_a, M, w_p, g_w, F, K, g_out, b)
    torch.cuda.synchronize()
    assert torch.equal(a.cpu(), b.cpu())
    # row 0 alone: an M = 1 call over the same prepared activation
    one = nv.act_buffer(F)
    nv.linear_swiglu(act16, g_a, 1, w_p, g_w, F, K, g_out, one)
    _, ref = _two_launches(act16, g_a, 1, w_p, g_w, F, K, g_out)
    torch.cuda.synchronize()
    assert torch.equal(one.cpu(), ref.cpu())
    assert nv.device_status() == (0, 0)


def test_fused_many_tiles_short_k():
    """Many gate tiles over a short K (F = 131,072, K = 512: each CTA sweeps
    the single K chunk several times), the shape where an activation-scale
    layout for repeated chunks would apply to a plain linear: the fused launch
    must stage every unit's scales and still equal the two-launch sequence
    (M = 4 keeps the reference quantiser's prepared image within its limit)."""
    cuda()
    M, F, K = 4, 131072, 512
    w_p, g_w, act, g_a = _operands(M, F, K, 11)
    g_out = torch.full((1,), 0.02, dtype=torch.float32, device="cuda")
    _, ref = _two_launches(act, g_a, M, w_p, g_w, F, K, g_out)
    fused = nv.act_buffer(F)
    nv.linear_swiglu(act, g_a, M, w_p, g_w, F, K, g_out, fused)
    torch.cuda.synchronize()
    assert nv.device_status() == (0, 0)
    assert torch.equal(fused.cpu(), ref.cpu())
