"""CPU pins of the element-wise quantiser check (tests/quant_check.py): a
correct alternative bf16 rounding at a near-midpoint element passes, and
planted mistakes (a wrong scale, a wrong code, a rounding flip where the
exact value is far from any midpoint) fail."""
import numpy as np
import pytest

from quant_check import DELTA, bf16_candidates, bf16_of, check_quant_bytes


def test_bf16_of_matches_torch():
    import torch
    x = np.random.default_rng(0).standard_normal(100000) * 3
    want = torch.from_numpy(x).float().to(torch.bfloat16).double().numpy()
    assert np.array_equal(bf16_of(x), want)


def test_candidates_only_near_midpoints():
    one_ulp = 2.0 ** -7                            # bf16 spacing on [1, 2)
    mid = 1.0 + one_ulp / 2                        # midpoint between 1 and 1 + 2^-7
    y = np.array([mid * (1 - 1e-7), mid * (1 + 1e-7), 1.0 + one_ulp / 4, mid * (1 + 1e-3), 0.0, -mid * (1 - 1e-7)])
    yb, nb = bf16_candidates(y)
    assert yb[0] == 1.0 and nb[0] == 1.0 + one_ulp
    assert yb[1] == 1.0 + one_ulp and nb[1] == 1.0
    assert np.isnan(nb[2]) and np.isnan(nb[3]) and np.isnan(nb[4])
    assert yb[5] == -1.0 and nb[5] == -(1.0 + one_ulp)


def _case(oracle, seed=1):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((4, 64))
    # element (1, 20) is the amax of its block and sits just below the midpoint
    # between the bf16 values 3 and 3 + 2^-6; g puts the block scale's E4M3
    # rounding midpoint (17, between 16 and 18) between the two, so the two
    # correct roundings give different scale bytes
    y[1, 16:32] *= 0.1
    y[1, 20] = (3.0 + 2.0 ** -6 / 2) * (1 - 1e-7)
    g = (3.0 + 2.0 ** -7) / (6 * 17)
    return y, g


def test_alternative_rounding_passes(oracle):
    y, g = _case(oracle)
    yb = bf16_of(y)
    alt = yb.copy()
    alt[1, 20] = 3.0 + 2.0 ** -6                    # the other neighbour
    c, s, _ = oracle.quantize(alt.astype(np.float32), g_in=g)
    c0, s0, _ = oracle.quantize(yb.astype(np.float32), g_in=g)
    assert not (np.array_equal(c, c0) and np.array_equal(s, s0)), "the flip must change the bytes"
    n_bad, _ = check_quant_bytes(oracle, y, c, s, g)
    assert n_bad == 1
    assert check_quant_bytes(oracle, y, c0, s0, g)[0] == 0


def test_planted_wrong_scale_fails(oracle):
    y, g = _case(oracle)
    c, s, _ = oracle.quantize(bf16_of(y).astype(np.float32), g_in=g)
    s = s.copy()
    s[2, 3] ^= 1                                   # block with no near-midpoint element
    with pytest.raises(AssertionError, match="no element"):
        check_quant_bytes(oracle, y, c, s, g)


def test_planted_wrong_code_in_ambiguous_block_fails(oracle):
    y, g = _case(oracle)
    c, s, _ = oracle.quantize(bf16_of(y).astype(np.float32), g_in=g)
    c = c.copy()
    c[1, 8 + 3] ^= 0x10                           # block 1 of row 1 holds the ambiguous element 20
    with pytest.raises(AssertionError, match="no correct bf16 rounding"):
        check_quant_bytes(oracle, y, c, s, g)


def test_flip_far_from_midpoint_fails(oracle):
    y, g = _case(oracle)
    yb = bf16_of(y)
    alt = yb.copy()
    j = int(np.argmax(np.abs(yb[2, :16])))          # the amax of block 0 of row 2 (no near-tie there)
    assert np.isnan(bf16_candidates(y)[1][2, :16]).all()
    alt[2, j] = bf16_of(yb[2, j] * 1.5)              # another bf16 value, far from the exact one
    c, s, _ = oracle.quantize(alt.astype(np.float32), g_in=g)
    c0, s0, _ = oracle.quantize(yb.astype(np.float32), g_in=g)
    assert not (np.array_equal(c, c0) and np.array_equal(s, s0))
    with pytest.raises(AssertionError):
        check_quant_bytes(oracle, y, c, s, g)
