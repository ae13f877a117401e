"""GPU parity of the many-token NVFP4 linear (the suffix prefill's linears):
tcgen05 block-scaled MMA over tiles of 128 weight rows x 256 tokens.

Bar: relative Frobenius error <= 1e-3 against bf16(fp64 oracle), as for the
skinny linear; whole outputs on small and ragged shapes, sampled outputs on
the prefill's layer shapes (942 suffix tokens), structured scale patterns
(each exercising one part of the scale-factor layout, the token side
included), the residual epilogue and determinism."""
import numpy as np
import pytest
import torch

from gpu_helpers import REL_FRO_TOL, bf16_round, cuda, host, rel_fro, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _prep(codes, scales, rows, K):
    return nv.prepare_weight(to_dev(codes), to_dev(scales), rows, K)


@pytest.mark.parametrize("mode", ["unit_scales", "row_scales", "kblock_scales", "token_scales", "random"])
def test_wide_scale_layout_structures(oracle, mode):
    cuda()
    rng = np.random.default_rng(60)
    S, N, K = 300, 256, 1024
    ac = rng.integers(0, 256, (S, K // 2), dtype=np.uint8)
    wc = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    one = 0x38
    asc = np.full((S, K // 16), one, np.uint8)
    wsc = np.full((N, K // 16), one, np.uint8)
    if mode == "row_scales":
        wsc[:] = rng.integers(0x30, 0x41, (N, 1))
    elif mode == "kblock_scales":
        wsc[:] = rng.integers(0x30, 0x41, (1, K // 16))
        asc[:] = rng.integers(0x30, 0x41, (1, K // 16))
    elif mode == "token_scales":
        asc[:] = rng.integers(0x30, 0x41, (S, 1))
    elif mode == "random":
        asc[:] = rng.integers(0x30, 0x41, (S, K // 16))
        wsc[:] = rng.integers(0x30, 0x41, (N, K // 16))
    gA, gW = 1.0, 0.5
    y = host(nv.linear_wide(_prep(ac, asc, S, K), to_dev(np.array([gA], np.float32)), S, _prep(wc, wsc, N, K),
                            to_dev(np.array([gW], np.float32)), N, K))
    want = oracle.linear(ac, asc, gA, wc, wsc, gW)
    err = rel_fro(y, bf16_round(want))
    assert err <= REL_FRO_TOL, f"{mode}: rel err {err:.3e}"


def _case(oracle, S, N, K, seed, full, residual=False, n_samples=6000):
    w = inputs.weight_fp32(70 + seed, 1, N, K)
    a = inputs.activation_bf16(70 + seed, 2, S, K, 0.01)
    owc, ows, ogw = oracle.quantize(w)
    oac, oas, oga = oracle.quantize(a.float().numpy())
    dw = to_dev(w)
    wc, wsc, gw = nv.quantize(dw)
    ac, asc, ga = nv.quantize(to_dev(a))
    assert np.array_equal(wc.cpu().numpy(), owc) and np.array_equal(asc.cpu().numpy(), oas)
    w_p = nv.prepare_weight(wc, wsc, N, K)
    a_p = nv.prepare_weight(ac, asc, S, K)
    res = inputs.bf16_normal(70 + seed, 3, (S, N)) if residual else None
    y = nv.linear_wide(a_p, ga, S, w_p, gw, N, K, residual=to_dev(res) if residual else None)
    got = host(y)
    if full:
        want = oracle.linear(oac, oas, oga, owc, ows, ogw)
        if residual:
            want = want + res.double().numpy()
        return rel_fro(got, bf16_round(want)), got, y
    rng = np.random.default_rng(seed)
    im, inn = rng.integers(0, S, n_samples), rng.integers(0, N, n_samples)
    want = oracle.linear_sampled(oac, oas, oga, owc, ows, ogw, im, inn)
    if residual:
        want = want + res.double().numpy()[im, inn]
    return rel_fro(got[im, inn], bf16_round(want)), got, y


@pytest.mark.parametrize("S,N,K", [(17, 256, 512), (128, 384, 1024), (129, 200, 640), (257, 130, 3072),
                                   (1, 128, 512), (100, 1000, 1536)])
def test_wide_small_shapes(oracle, S, N, K):
    """Whole outputs, ragged in S (token tiles of 128 / 256), N and K."""
    cuda()
    err, _, _ = _case(oracle, S, N, K, S + N, full=True)
    assert err <= REL_FRO_TOL, err


@pytest.mark.parametrize("name", ["qkv", "o", "gate_up", "down"])
def test_wide_prefill_layer_shapes(oracle, name):
    """The layer's four linears over the 942-token suffix, sampled outputs."""
    cuda()
    K, N = inputs.LAYER_LINEARS[name]
    err, _, _ = _case(oracle, 942, N, K, {"qkv": 1, "o": 2, "gate_up": 3, "down": 4}[name], full=False)
    assert err <= REL_FRO_TOL, err


def test_wide_residual_and_determinism(oracle):
    cuda()
    err, got, y = _case(oracle, 300, 512, 1024, 9, full=True, residual=True)
    assert err <= REL_FRO_TOL, err
    # same call again: bit-identical
    err2, got2, _ = _case(oracle, 300, 512, 1024, 9, full=True, residual=True)
    assert np.array_equal(got, got2)
    assert nv.device_status()[0] == 0
