"""Pins for the oracle's codecs (E2M1 per OCP MX v1.0, E4M3 per OCP OFP8).

The oracle builds both tables from the bit fields; these tests pin them to
fixed facts of the specifications, to torch's own float8_e4m3fn type, and
pin the RNE/satfinite encoders to numpy's round-half-even (np.rint) and to
torch's float32 -> float8_e4m3fn cast.
"""
import math

import numpy as np
import torch

# E2M1 magnitudes for codes 0..7 as listed in the OCP MX v1.0 FP4 table.
E2M1_SPEC = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_table_is_the_spec_table(oracle):
    t = oracle.e2m1_table()
    assert t.shape == (16,)
    assert list(t[:8]) == E2M1_SPEC
    assert list(-t[8:]) == E2M1_SPEC
    assert t[0x7] == 6.0 and t[0xF] == -6.0
    assert math.copysign(1.0, t[0x8]) == -1.0 and t[0x8] == 0.0   # 0x8 is -0


def test_e4m3_anchors(oracle):
    t = oracle.e4m3_table()
    assert t.shape == (256,)
    assert t[0x7E] == 448.0
    assert t[0x08] == 2.0 ** -6          # smallest normal
    assert t[0x01] == 2.0 ** -9          # smallest subnormal
    assert t[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert t[0x38] == 1.0
    assert t[0x00] == 0.0 and math.copysign(1.0, t[0x80]) == -1.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert t[0xFE] == -448.0
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must be strictly increasing"
    assert np.array_equal(t[0x80:0xFF], -t[:0x7F])


def test_e4m3_table_matches_torch_float8(oracle):
    t = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    finite = ~np.isnan(t)
    assert np.array_equal(np.isnan(ref), ~finite)
    assert np.array_equal(t[finite], ref[finite])


def _e2m1_rint_reference(v):
    """E2M1 RNE+satfinite via np.rint (round-half-even) on each binade."""
    a = abs(v)
    if a <= 2.0:
        code = int(np.rint(2.0 * a))                      # spacing 0.5: codes 0..4
    elif a <= 4.0:
        code = 4 + int(np.rint(a)) - 2                    # spacing 1: codes 4..6
    elif a < 6.0:
        code = 6 + (int(np.rint(a / 2.0)) - 2)            # spacing 2: codes 6..7
    else:
        code = 7
    return code | (8 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_encoder_ties_and_saturation(oracle):
    # ties go to the even code (mantissa bit 0)
    cases = [(0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
             (5.0, 0x6), (6.0, 0x7), (7.0, 0x7), (1e30, 0x7), (0.0, 0x0), (-0.0, 0x8),
             (-0.1, 0x8), (-5.0, 0xE)]
    for v, c in cases:
        assert oracle.e2m1_encode(v) == c, v


def test_e2m1_encoder_matches_rint_binades(oracle):
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(-8, 8, 4000)) + [m + s for m in np.arange(-7, 7.25, 0.25)
                                             for s in (-1e-7, 0.0, 1e-7)]
    for v in vals:
        v32 = float(np.float32(v))
        assert oracle.e2m1_encode(v32) == _e2m1_rint_reference(v32), v32


def test_e4m3_encoder_matches_torch_cast(oracle):
    rng = np.random.default_rng(2)
    t = oracle.e4m3_table()
    mids = (t[:0x7E] + t[1:0x7F]) / 2.0           # exact ties between neighbours
    vals = np.concatenate([
        rng.uniform(-448, 448, 20000),
        np.exp2(rng.uniform(-12, 8.8, 20000)) * rng.choice([-1, 1], 20000),
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1000),
    ]).astype(np.float32)
    vals = vals[np.abs(vals) <= 448]
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    _, ours = oracle.encode_many(vals)
    assert np.array_equal(ours, ref)


def test_e4m3_encoder_saturates(oracle):
    for v, c in {448.0: 0x7E, 463.9: 0x7E, 464.0: 0x7E, 500.0: 0x7E, 1e38: 0x7E, -1e38: 0xFE,
                 2.0 ** -10: 0x00, 2.0 ** -10 * 1.0001: 0x01, 3 * 2.0 ** -10: 0x02}.items():
        assert oracle.e4m3_encode(v) == c, v
