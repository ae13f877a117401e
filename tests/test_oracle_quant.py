"""Pins for the oracle's NVFP4 quantiser and W4A4 linear layer.

Quantiser: the hand-worked example in tests/golden, exact round trips of
values on the E2M1 grid times an exact E4M3 scale, the zero-block and
zero-tensor readings, the independence of a block from every other block
except through the tensor scale, and agreement with the same fp32 recipe
evaluated by numpy float32 arithmetic + torch's float8 cast + np.rint.

Linear: a one-block closed form, and numpy fp64 matmul of operands
dequantised here (torch float8 view for scales, the spec's E2M1 list for
codes) on a tiny shape; row independence.
"""
import json
import math
import os

import numpy as np
import torch

from test_oracle_codecs import E2M1_SPEC, _e2m1_rint_reference

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example(oracle):
    ex = json.load(open(os.path.join(GOLDEN, "nvfp4_quant_worked_example.json")))
    x = np.array(ex["x"], np.float32).reshape(1, -1)
    codes, scales, g = oracle.quantize(x)
    assert g == ex["g"]
    assert [f"{b:02X}" for b in scales.ravel()] == ex["scales_hex"]
    assert [f"{b:02X}" for b in codes.ravel()] == ex["codes_hex"]


def _e4m3_value(code):
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).double())


def test_grid_values_round_trip_exactly(oracle):
    rng = np.random.default_rng(3)
    grid = np.array(E2M1_SPEC[1:] + [-v for v in E2M1_SPEC[1:]])
    for g_in in (1.0, 0.25, 8.0):
        rows, K = 4, 64
        x = np.zeros((rows, K), np.float64)
        want_sc = rng.integers(0x08, 0x7F, size=(rows, K // 16))
        for r in range(rows):
            for b in range(K // 16):
                S = _e4m3_value(int(want_sc[r, b]))
                c = rng.choice(grid, 16)
                c[rng.integers(16)] = rng.choice([6.0, -6.0])      # block amax = 6 S g
                x[r, b * 16:(b + 1) * 16] = c * S * g_in
        x32 = x.astype(np.float32)
        assert np.array_equal(x32.astype(np.float64), x)
        codes, scales, g = oracle.quantize(x32, g_in=g_in)
        assert g == g_in
        assert np.array_equal(scales, want_sc.astype(np.uint8))
        assert np.array_equal(oracle.dequantize(codes, scales, g), x)


def test_zero_block_and_zero_tensor(oracle):
    x = np.zeros((2, 32), np.float32)
    x[0, 16:] = np.linspace(-1, 1, 16)
    x[1, :16] = -0.0
    codes, scales, g = oracle.quantize(x)
    assert scales[0, 0] == 0 and scales[1, 0] == 0
    assert np.all(codes[0, :8] == 0) and np.all(codes[1, :8] == 0)   # s == 0 -> +0 codes
    _, _, g0 = oracle.quantize(np.zeros((3, 16), np.float32))
    assert g0 == 1.0                                                  # reading: amax == 0 -> g = 1


def test_tensor_scale_closed_form(oracle):
    x = np.zeros((1, 16), np.float32)
    x[0, 5] = -2688.0
    assert oracle.tensor_scale(x) == 1.0
    x[0, 5] = 1.0
    assert oracle.tensor_scale(x) == float(np.float32(1.0) / np.float32(2688.0))


def test_blocks_interact_only_through_g(oracle):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 128)).astype(np.float32)
    x[1, 40] = 300.0                                                 # single outlier block
    codes, scales, g = oracle.quantize(x)
    for r in range(3):
        for b in range(8):
            blk = x[r:r + 1, b * 16:(b + 1) * 16]
            c1, s1, _ = oracle.quantize(blk, g_in=g)
            assert s1[0, 0] == scales[r, b]
            assert np.array_equal(c1[0], codes[r, b * 8:(b + 1) * 8])


def _recipe_numpy(x):
    """The fp32 recipe evaluated with numpy float32 ops, torch's E4M3 cast and
    np.rint-based E2M1 rounding (independent of the oracle's C code)."""
    x = x.astype(np.float32)
    amax = np.float32(np.abs(x).max())
    g = np.float32(amax / np.float32(2688.0)) if amax > 0 else np.float32(1.0)
    rows, K = x.shape
    scales = np.zeros((rows, K // 16), np.uint8)
    codes = np.zeros((rows, K), np.uint8)
    for r in range(rows):
        for b in range(K // 16):
            blk = x[r, b * 16:(b + 1) * 16]
            rr = np.float32(np.float32(np.abs(blk).max()) / np.float32(6.0))
            t = np.float32(rr / g)
            t = min(float(t), 448.0)
            sc = int(torch.tensor([t], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8))
            scales[r, b] = sc
            s = np.float32(np.float32(_e4m3_value(sc)) * g)
            for k in range(16):
                codes[r, b * 16 + k] = 0 if s == 0 else _e2m1_rint_reference(float(np.float32(blk[k] / s)))
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, scales, float(g)


def test_matches_fp32_recipe_evaluated_by_numpy(oracle):
    rng = np.random.default_rng(5)
    for trial in range(6):
        x = rng.standard_normal((3, 64)).astype(np.float32) * np.float32(10.0 ** rng.uniform(-6, 4))
        if trial % 2:
            x[:, rng.integers(64)] *= 20.0                          # outlier channel
        want = _recipe_numpy(x)
        got = oracle.quantize(x)
        assert got[2] == want[2]
        assert np.array_equal(got[1], want[1])
        assert np.array_equal(got[0], want[0])


# ------------------------------------------------------------------ linear
def _dequant_here(codes, scales, g):
    e2 = np.array(E2M1_SPEC + [-v for v in E2M1_SPEC])
    rows = codes.shape[0]
    vals = np.empty((rows, codes.shape[1] * 2))
    vals[:, 0::2] = e2[codes & 15]
    vals[:, 1::2] = e2[codes >> 4]
    sv = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy()
    return float(g) * vals * np.repeat(sv, 16, axis=1)


def test_linear_one_block_closed_form(oracle):
    K = 64
    a_codes = np.zeros((1, K // 2), np.uint8)
    w_codes = np.zeros((1, K // 2), np.uint8)
    a_codes[0, 8:16] = 0x22          # block 1: sixteen 1.0s
    w_codes[0, 8:16] = 0x22
    a_sc = np.zeros((1, 4), np.uint8); a_sc[0, 1] = 0x38    # 1.0
    w_sc = np.zeros((1, 4), np.uint8); w_sc[0, 1] = 0x40    # 2.0
    y = oracle.linear(a_codes, a_sc, 1.0, w_codes, w_sc, 0.5)
    assert y[0, 0] == 1.0 * 0.5 * (1.0 * 2.0) * 16


def test_linear_tiny_bruteforce_vs_numpy_matmul(oracle):
    rng = np.random.default_rng(6)
    M, N, K = 2, 8, 64
    a = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    ac, asc, ga = oracle.quantize(a)
    wc, wsc, gw = oracle.quantize(w)
    want = _dequant_here(ac, asc, ga) @ _dequant_here(wc, wsc, gw).T
    got = oracle.linear(ac, asc, ga, wc, wsc, gw)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
    # and the dequantiser agrees with the independent one
    assert np.array_equal(oracle.dequantize(ac, asc, ga), _dequant_here(ac, asc, ga))


def test_linear_rows_are_independent(oracle):
    rng = np.random.default_rng(7)
    a = rng.standard_normal((16, 256)).astype(np.float32)
    w = (rng.standard_normal((24, 256)) * 0.02).astype(np.float32)
    wc, wsc, gw = oracle.quantize(w)
    ac, asc, ga = oracle.quantize(a, g_in=0.01)
    full = oracle.linear(ac, asc, ga, wc, wsc, gw)
    for m in (0, 7, 15):
        one = oracle.linear(ac[m:m + 1], asc[m:m + 1], ga, wc, wsc, gw)
        assert np.array_equal(one[0], full[m])
    idx_m = np.array([0, 3, 15, 15]); idx_n = np.array([0, 5, 23, 1])
    s = oracle.linear_sampled(ac, asc, ga, wc, wsc, gw, idx_m, idx_n)
    assert np.array_equal(s, full[idx_m, idx_n])
