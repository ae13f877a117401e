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


def _bf16_values(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("g", [1e-3, 0.0037913, 3.7, 1e-30, 2.0 ** -120])
def test_division_every_bf16_dividend_every_scale(oracle, g):
    """The quantiser's element division x / s, exhaustively over bf16
    dividends: for every positive finite E4M3 scale code (and a few amax
    values that saturate the scale), blocks whose first element A sets the
    block scale and whose other 15 elements run through every bf16 value of
    magnitude <= A, both signs.  Codes and scales must equal the oracle's
    (correctly rounded fp32 division) bit for bit.  Covers the reciprocal +
    correction path and, with the tiny tensor scales, its exact-division
    fallback (scales below 2^-100)."""
    cuda()
    e4 = oracle.e4m3_table()[1:0x7F].astype(np.float64)
    amaxes = list(e4 * 6.0 * g) + [448.0 * 6.0 * g * 2.0 ** k for k in (1, 10, 60, 110)]
    blocks = []
    for A in amaxes:
        A32 = np.float32(A)
        if not np.isfinite(A32) or A32 == 0:
            continue
        a_bits = int(np.float32(A32).view(np.uint32)) >> 16          # bf16 at or below A
        vals = _bf16_values(np.arange(0, a_bits + 1))
        vals = np.stack([vals, -vals], 1).ravel()
        n = -(-vals.size // 15) * 15
        vals = np.concatenate([vals, np.zeros(n - vals.size, np.float32)]).reshape(-1, 15)
        head = np.full((vals.shape[0], 1), _bf16_values([a_bits])[0], np.float32)
        blocks.append(np.concatenate([head, vals], 1))
    x = np.concatenate(blocks).ravel()
    K = 16384
    x = np.concatenate([x, np.zeros(-x.size % K, np.float32)]).reshape(-1, K)
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    assert np.array_equal(xd.float().cpu().numpy(), x)               # every value is a bf16
    codes, scales, _ = nv.quantize(xd, g_in=to_dev(np.array([g], np.float32)))
    torch.cuda.synchronize()
    oc, osc, _ = oracle.quantize(x, g_in=g)
    gs, gc = scales.cpu().numpy(), codes.cpu().numpy()
    bad_s = np.argwhere(gs != osc)
    assert bad_s.size == 0, f"{len(bad_s)} scale mismatches, first {bad_s[:5].tolist()}"
    bad_c = np.argwhere(gc != oc)
    assert bad_c.size == 0, f"{len(bad_c)} code-byte mismatches, first {bad_c[:5].tolist()}"
    assert len(np.unique(osc)) >= 100                                 # the sweep reaches the scale codes
    print(f"g={g}: {x.size} elements, {len(np.unique(osc))} scale codes")


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


def test_prepare_weight_layout():
    """Prepared weight units: per (128-row tile, 512-K chunk), two 128-byte-
    swizzled 16 KB code atoms then eight 512-byte scale images (line l, byte
    4c + kb = scale of row l + 32c, block 4j + kb); zero-padded."""
    cuda()
    rng = np.random.default_rng(34)
    for N, K in [(128, 512), (200, 576), (300, 1024)]:
        codes = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
        sc = rng.integers(0, 0x7F, (N, K // 16), dtype=np.uint8)
        prep = nv.prepare_weight(to_dev(codes), to_dev(sc), N, K).cpu().numpy()
        NT, KC = -(-N // 128), -(-K // 512)
        unit = 36864
        want = np.zeros(NT * KC * unit, np.uint8)
        for t in range(NT):
            for c in range(KC):
                base = (t * KC + c) * unit
                for a in range(2):
                    for r in range(128):
                        row = t * 128 + r
                        for b in range(128):
                            col = c * 256 + a * 128 + b
                            if row < N and col < K // 2:
                                want[base + a * 16384 + r * 128 + ((((b >> 4) ^ (r & 7)) << 4) | (b & 15))] = codes[row, col]
                for j in range(8):
                    for l in range(32):
                        for cc in range(4):
                            for kb in range(4):
                                row, blk = t * 128 + l + 32 * cc, c * 32 + 4 * j + kb
                                if row < N and blk < K // 16:
                                    want[base + 32768 + j * 512 + l * 16 + 4 * cc + kb] = sc[row, blk]
        assert np.array_equal(prep, want)


def test_conversion_every_finite_fp32(oracle):
    """fp32 -> E2M1 and fp32 -> E4M3 (round-to-nearest-even, saturating, sign
    kept) on every finite fp32 bit pattern, both signs: the device conversion
    instructions the quantisers use against the oracle's decision rule."""
    cuda()
    chunk = 1 << 26
    bad2 = bad4 = 0
    first = None
    for sign in (0, 0x80000000):
        for start in range(0, 0x7F800000, chunk):
            n = min(chunk, 0x7F800000 - start)
            pats = np.arange(sign + start, sign + start + n, dtype=np.uint64).astype(np.uint32)
            x = pats.view(np.float32)
            ge2, ge4 = nv.debug_encode(to_dev(x))
            oe2, oe4 = oracle.encode_many(x)
            d2 = np.flatnonzero(ge2.cpu().numpy() != oe2)
            d4 = np.flatnonzero(ge4.cpu().numpy() != oe4)
            bad2 += d2.size
            bad4 += d4.size
            if first is None and (d2.size or d4.size):
                first = hex(int(pats[(d2 if d2.size else d4)[0]]))
    assert bad2 == 0 and bad4 == 0, (bad2, bad4, first)
