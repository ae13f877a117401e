"""GPU parity of the NVFP4 linear layer (tcgen05 block-scaled MMA, split-K).

Bar: relative Frobenius error <= 1e-3 against bf16(fp64 oracle), on the
shapes of the single-linear, layer and LM-head workloads, ragged shapes,
structured scale patterns (each exercising one part of the scale-factor
layout), row independence (bit-identical rows between M=16 and M=1 calls),
determinism, the residual epilogue and the LM-head argmax rule."""
import numpy as np
import pytest
import torch

from gpu_helpers import REL_FRO_TOL, bf16_round, cuda, host, rel_fro, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _gpu_operands(codes, scales, g, N, K):
    c, s = to_dev(codes), to_dev(scales)
    return c, s, to_dev(np.array([g], np.float32)), nv.prepare_weight(c, s, N, K)


@pytest.mark.parametrize("mode", ["unit_scales", "row_scales", "kblock_scales", "token_scales", "random"])
def test_scale_layout_structures(oracle, mode):
    """Random E2M1 codes with structured scales: each mode isolates one part of
    the operand / scale-factor layout, so a failure names the broken part."""
    cuda()
    rng = np.random.default_rng(40)
    M, N, K = 16, 256, 512
    ac = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    wc = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    one = 0x38
    asc = np.full((M, K // 16), one, np.uint8)
    wsc = np.full((N, K // 16), one, np.uint8)
    if mode == "row_scales":
        wsc[:] = rng.integers(0x30, 0x41, (N, 1))
    elif mode == "kblock_scales":
        wsc[:] = rng.integers(0x30, 0x41, (1, K // 16))
        asc[:] = rng.integers(0x30, 0x41, (1, K // 16))
    elif mode == "token_scales":
        asc[:] = rng.integers(0x30, 0x41, (M, 1))
    elif mode == "random":
        asc[:] = rng.integers(0x30, 0x41, (M, K // 16))
        wsc[:] = rng.integers(0x30, 0x41, (N, K // 16))
    gA, gW = 1.0, 0.5
    a_c, a_s, a_g = to_dev(ac), to_dev(asc), to_dev(np.array([gA], np.float32))
    a_p = nv.prepare_act(a_c, a_s, K)
    w_c, _, w_g, w_p = _gpu_operands(wc, wsc, gW, N, K)
    y = host(nv.linear(a_p, a_g, M, w_p, w_g, N, K))
    want = oracle.linear(ac, asc, gA, wc, wsc, gW)
    err = rel_fro(y, bf16_round(want))
    assert err <= REL_FRO_TOL, f"{mode}: rel err {err:.3e}"


def _case(oracle, M, N, K, outliers, seed, full=True, n_samples=8192):
    w = inputs.weight_fp32(50 + seed, 1, N, K)
    a = inputs.activation_bf16(50 + seed, 2, M, K, outliers)
    owc, ows, ogw = oracle.quantize(w)
    oac, oas, oga = oracle.quantize(a.float().numpy())
    wc, ws, gw = nv.quantize(to_dev(w))
    act = nv.act_buffer(K)
    ac, asc, ga = nv.quantize(to_dev(a), act=act)
    assert np.array_equal(wc.cpu().numpy(), owc) and np.array_equal(ws.cpu().numpy(), ows)
    assert np.array_equal(ac.cpu().numpy(), oac) and np.array_equal(asc.cpu().numpy(), oas)
    wp = nv.prepare_weight(wc, ws, N, K)
    y = nv.linear(act, ga, M, wp, gw, N, K)
    ops = (act, ga, M, wp, gw)
    if full:
        want = oracle.linear(oac, oas, oga, owc, ows, ogw)
        return host(y), want, ops
    rng = np.random.default_rng(seed)
    im = rng.integers(0, M, n_samples)
    inn = rng.integers(0, N, n_samples)
    want = oracle.linear_sampled(oac, oas, oga, owc, ows, ogw, im, inn)
    return host(y)[im, inn], want, ops


@pytest.mark.parametrize("name,M,N,K,outl", [
    ("single_M1_2048", 1, 2048, 2048, 0.0),
    ("qkv", 16, 4096, 5120, 0.01),
    ("o_proj", 16, 5120, 3072, 0.01),
    ("ragged", 3, 200, 320, 0.0),
    ("ragged2", 16, 1000, 576, 0.01),
    ("tiny_K", 5, 130, 64, 0.0),
])
def test_linear_full_parity(oracle, name, M, N, K, outl):
    cuda()
    y, want, _ = _case(oracle, M, N, K, outl, seed=sum(map(ord, name)))
    err = rel_fro(y, bf16_round(want))
    assert err <= REL_FRO_TOL, f"{name}: rel err {err:.3e}"


@pytest.mark.parametrize("name,M,N,K", [("gate_up", 16, 34816, 5120), ("down", 16, 5120, 17408)])
def test_linear_layer_shapes_sampled(oracle, name, M, N, K):
    cuda()
    y, want, _ = _case(oracle, M, N, K, 0.01, seed=7 + K % 97, full=False)
    err = rel_fro(y, bf16_round(want))
    assert err <= REL_FRO_TOL, f"{name}: rel err {err:.3e}"


def test_rows_independent_and_deterministic(oracle):
    cuda()
    M, N, K = 16, 4096, 5120
    w = inputs.weight_fp32(60, 1, N, K)
    a = inputs.activation_bf16(60, 2, M, K, 0.01)
    wc, ws, gw = nv.quantize(to_dev(w))
    wp = nv.prepare_weight(wc, ws, N, K)
    gin = to_dev(np.array([0.01], np.float32))
    ad = to_dev(a)
    act = nv.act_buffer(K)
    _, _, ga = nv.quantize(ad, g_in=gin, act=act)
    y16 = nv.linear(act, ga, M, wp, gw, N, K).clone()
    y16b = nv.linear(act, ga, M, wp, gw, N, K).clone()
    assert torch.equal(y16, y16b)
    for m in (0, 9, 15):
        act1 = nv.act_buffer(K)
        _, _, g1 = nv.quantize(ad[m:m + 1], g_in=gin, act=act1)
        y1 = nv.linear(act1, g1, 1, wp, gw, N, K)
        assert torch.equal(y1[0], y16[m]), m


def test_linear_split_grid_invariance(oracle):
    """Different split-K grids give the same result up to fp32 summation order."""
    cuda()
    M, N, K = 16, 1024, 5120
    _, _, ops = _case(oracle, M, N, K, 0.01, seed=61, full=False, n_samples=16)
    act, ga, M, wp, gw = ops
    ref = host(nv.linear(act, ga, M, wp, gw, N, K))
    try:
        for G in (1, 7, 33, 160):
            nv.set_option(nv.OPT_LINEAR_CTAS, G)
            y = host(nv.linear(act, ga, M, wp, gw, N, K))
            assert rel_fro(y, ref) < 1e-5, G
    finally:
        nv.set_option(nv.OPT_LINEAR_CTAS, 0)


def test_residual_epilogue(oracle):
    cuda()
    M, N, K = 16, 640, 1024
    y, want, ops = _case(oracle, M, N, K, 0.0, seed=62)
    act, ga, M, wp, gw = ops
    res = inputs.bf16_normal(62, 5, (M, N))
    out = to_dev(res).clone()
    nv.linear(act, ga, M, wp, gw, N, K, y=out, residual=out)     # in place
    err = rel_fro(host(out), bf16_round(want + res.double().numpy()))
    assert err <= REL_FRO_TOL


@pytest.mark.parametrize("M", [1, 16])
def test_lm_head_argmax(oracle, M):
    """LM head (N = 151936): sampled logits within the GEMM bar, and the argmax
    of every row equals the oracle's where top1 - top2 > tau, tau =
    ulp_bf16(|top1|) + 1e-4 |top1|."""
    cuda()
    N, K = inputs.VOCAB, inputs.HIDDEN
    w = inputs.weight_fp32(2, 1, N, K)
    a = inputs.activation_bf16(2, 2, M, K, 0.0)
    owc, ows, ogw = oracle.quantize(w)
    oac, oas, oga = oracle.quantize(a.float().numpy())
    wc, ws, gw = nv.quantize(to_dev(w))
    del w
    assert np.array_equal(ws.cpu().numpy(), ows)
    assert np.array_equal(wc.cpu().numpy(), owc)
    act = nv.act_buffer(K)
    _, _, ga = nv.quantize(to_dev(a), act=act)
    wp = nv.prepare_weight(wc, ws, N, K)
    del wc, ws
    y = nv.linear(act, ga, M, wp, gw, N, K)
    idx = nv.argmax(y).cpu().numpy()
    yh = host(y)
    want = oracle.linear(oac, oas, oga, owc, ows, ogw)
    assert rel_fro(yh, bf16_round(want)) <= REL_FRO_TOL
    for m in range(M):
        srt = np.sort(want[m])
        top1, top2 = srt[-1], srt[-2]
        tau = np.spacing(np.float32(abs(top1))) * 2 ** 16 + 1e-4 * abs(top1)   # bf16 ulp = fp32 ulp * 2^16
        # the GPU's argmax is the argmax of its own bf16 logits (lowest index on ties)
        assert idx[m] == int(np.argmax(yh[m])), m
        if top1 - top2 > tau:
            assert idx[m] == int(np.argmax(want[m])), (m, top1, top2)


def test_linear_rejects_bad_arguments():
    cuda()
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    g = torch.ones(1, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:          # M > 16
        nv._call("nvfp4_linear", z.data_ptr(), g.data_ptr(), 17, z.data_ptr(), g.data_ptr(), 8, 64, None,
                 z.data_ptr(), 8, z.data_ptr(), 1 << 16, 0)
    assert e.value.code == -2
    with pytest.raises(nv.NvFp4Error) as e:          # misaligned prepared activation
        nv._call("nvfp4_linear", z.data_ptr() + 1, g.data_ptr(), 1, z.data_ptr(), g.data_ptr(), 8, 64, None,
                 z.data_ptr(), 8, z.data_ptr(), 1 << 16, 0)
    assert e.value.code == -3
    with pytest.raises(nv.NvFp4Error) as e:          # workspace too small
        nv._call("nvfp4_linear", z.data_ptr(), g.data_ptr(), 1, z.data_ptr(), g.data_ptr(), 8, 64, None,
                 z.data_ptr(), 8, z.data_ptr(), 16, 0)
    assert e.value.code == -4


@pytest.mark.parametrize("M,K", [(16, 5120), (3, 576), (1, 64)])
def test_prepared_activation_layout(M, K):
    """quantize(act=...) writes exactly the re-layout of its canonical outputs,
    which follows the documented tile image; untouched bytes stay zero."""
    cuda()
    a = inputs.activation_bf16(63, 0, M, K, 0.01)
    act = nv.act_buffer(K)
    codes, scales, g = nv.quantize(to_dev(a), act=act)
    act2 = nv.prepare_act(codes, scales, K)
    assert torch.equal(act, act2)
    c, sc = codes.cpu().numpy(), scales.cpu().numpy()
    want = np.zeros(act.numel(), np.uint8)
    for m in range(M):
        for blk in range(K // 16):
            cidx, bi = blk // 32, blk % 32
            base = cidx * 8192
            b = (bi % 16) * 8
            off = base + (bi // 16) * 2048 + m * 128 + ((((b >> 4) ^ (m & 7)) << 4) | (b & 15))
            want[off:off + 8] = c[m, blk * 8:blk * 8 + 8]
            want[base + 4096 + (bi // 4) * 512 + m * 16 + bi % 4] = sc[m, blk]
    assert np.array_equal(act.cpu().numpy(), want)


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_linear_every_row_count(oracle, M):
    """Every token count 1..16 (rows past M of the prepared activation are
    zero; outputs past M are never written), whole outputs on a ragged shape."""
    cuda()
    y, want, _ = _case(oracle, M, 384, 1088, 0.01, seed=100 + M)
    err = rel_fro(y, bf16_round(want))
    assert err <= REL_FRO_TOL, f"M={M}: rel err {err:.3e}"
