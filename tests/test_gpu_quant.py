"""GPU parity of the NVFP4 quantiser: bit-exact codes, scales and tensor scale
against the oracle, on the activation and weight shapes of the workloads,
ragged and degenerate inputs, and a sweep of the fp32 -> E2M1/E4M3
conversions."""
import numpy as np
import pytest
import torch

from gpu_helpers import cuda, to_dev
from nvfp4_skinny_gemm_b200 import inputs
from nvfp4_skinny_gemm_b200 import lib as nv

pytestmark = pytest.mark.gpu


def _check_bitexact(oracle, x_host_f32, x_dev, g_in=None):
    codes, scales, g = nv.quantize(x_dev, g_in=None if g_in is None else to_dev(np.array([g_in], np.float32)))
    torch.cuda.synchronize()
    oc, osc, og = oracle.quantize(x_host_f32, g_in=g_in)
    gc, gs, gg = codes.cpu().numpy(), scales.cpu().numpy(), float(g.cpu()[0])
    assert gg == og, (gg, og)
    bad_s = np.argwhere(gs != osc)
    assert bad_s.size == 0, f"{len(bad_s)} scale mismatches, first {bad_s[:5].tolist()}"
    bad_c = np.argwhere(gc != oc)
    assert bad_c.size == 0, f"{len(bad_c)} code-byte mismatches, first {bad_c[:5].tolist()}"


def test_conversion_sweep_matches_oracle(oracle):
    cuda()
    rng = np.random.default_rng(21)
    e2 = oracle.e2m1_table()[:8]
    e4 = oracle.e4m3_table()[:0x7F]
    ties2 = (e2[:-1] + e2[1:]) / 2
    ties4 = (e4[:-1] + e4[1:]) / 2
    base = np.concatenate([
        ties2, ties4, e2, e4,
        np.nextafter(ties2, 0), np.nextafter(ties2, 10), np.nextafter(ties4, 0), np.nextafter(ties4, 1000),
        [0.0, 1e-45, 1e-38, 6.0, 6.5, 7.0, 448.0, 464.0, 480.0, 1e4, 1e38, np.float32(3.4e38)],
        rng.uniform(0, 8, 1 << 20), np.exp2(rng.uniform(-40, 12, 1 << 20)),
    ])
    # every fp32 bit pattern of [0.25, 8) with a stride, plus the subnormal E4M3 range densely
    lo, hi = np.float32(0.25).view(np.uint32), np.float32(8.0).view(np.uint32)
    pats = np.arange(lo, hi, 97, dtype=np.uint32).view(np.float32)
    lo4, hi4 = np.float32(2.0 ** -11).view(np.uint32), np.float32(2.0 ** -5).view(np.uint32)
    pats4 = np.arange(lo4, hi4, 61, dtype=np.uint32).view(np.float32)
    x = np.concatenate([base, -base, pats, -pats, pats4]).astype(np.float32)
    x[0] = -0.0
    ge2, ge4 = nv.debug_encode(to_dev(x))
    oe2, oe4 = oracle.encode_many(x)
    ge2, ge4 = ge2.cpu().numpy(), ge4.cpu().numpy()
    bad2 = np.flatnonzero(ge2 != oe2)
    bad4 = np.flatnonzero(ge4 != oe4)
    assert bad2.size == 0, f"E2M1: {bad2.size} mismatches, e.g. x={x[bad2[:4]]} gpu={ge2[bad2[:4]]} oracle={oe2[bad2[:4]]}"
    assert bad4.size == 0, f"E4M3: {bad4.size} mismatches, e.g. x={x[bad4[:4]]} gpu={ge4[bad4[:4]]} oracle={oe4[bad4[:4]]}"


@pytest.mark.parametrize("M,K,outliers", [(1, 2048, 0.0), (16, 5120, 0.01), (16, 3072, 0.01),
                                          (16, 17408, 0.01), (3, 80, 0.0), (16, 34816, 0.0)])
def test_activation_bf16_bitexact(oracle, M, K, outliers):
    cuda()
    a = inputs.activation_bf16(30, K, M, K, outliers)
    _check_bitexact(oracle, a.float().numpy(), to_dev(a))


def test_activation_static_scale(oracle):
    cuda()
    a = inputs.activation_bf16(31, 0, 16, 5120, 0.01)
    _check_bitexact(oracle, a.float().numpy(), to_dev(a), g_in=0.0137)


@pytest.mark.parametrize("N,K", [(2048, 2048), (4096, 5120), (300, 17408)])
def test_weight_fp32_bitexact(oracle, N, K):
    cuda()
    w = inputs.weight_fp32(32, 1, N, K)
    _check_bitexact(oracle, w, to_dev(w))


def test_large_bf16_two_kernel_path(oracle):
    cuda()
    a = inputs.activation_bf16(33, 0, 600, 1024, 0.01)    # > fused-path capacity
    _check_bitexact(oracle, a.float().numpy(), to_dev(a))
    _check_bitexact(oracle, a.float().numpy(), to_dev(a), g_in=0.25)


def test_degenerate_inputs(oracle):
    cuda()
    z = np.zeros((2, 64), np.float32)
    _check_bitexact(oracle, z, to_dev(z))                  # all zero: g = 1, scales 0, codes 0
    x = np.zeros((4, 64), np.float32)
    x[1, 17] = -3.0
    x[2, :16] = -0.0
    x[3, 40:48] = 1e-30
    _check_bitexact(oracle, x, to_dev(x))
    t = torch.zeros(16, 4096, dtype=torch.bfloat16)
    t[5, 100] = 1.0
    _check_bitexact(oracle, t.float().numpy(), to_dev(t))


def test_rejects_bad_shapes():
    cuda()
    x = torch.zeros(2, 24, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.quantize(x)
    assert e.value.code == -2


def test_prepare_scales_layout():
    cuda()
    rng = np.random.default_rng(34)
    for N, K in [(128, 256), (200, 320), (384, 5120)]:
        sc = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
        prep = nv.prepare_weight_scales(to_dev(sc), N, K).cpu().numpy()
        NT, KT = -(-N // 128), -(-K // 256)
        want = np.zeros((NT, KT, 4, 32, 4, 4), np.uint8)     # [t][kt][j][l][c][kb]
        for t in range(NT):
            for kt in range(KT):
                for j in range(4):
                    for c in range(4):
                        rows = t * 128 + np.arange(32) + 32 * c
                        for kb in range(4):
                            col = kt * 16 + 4 * j + kb
                            ok = (rows < N) & (col < K // 16)
                            want[t, kt, j, :, c, kb] = np.where(ok, sc[np.minimum(rows, N - 1), min(col, K // 16 - 1)], 0)
        assert np.array_equal(prep, want.ravel())
