"""Element-wise parity of a fused "op -> bf16 -> NVFP4" kernel against the oracle.

A fused quantiser (RMSNorm or SwiGLU followed by NVFP4) rounds its fp32 op
output to bf16 and quantises that.  The oracle computes the op in fp64, rounds
to bf16 and quantises.  Where the exact value lies so close to the midpoint
between two bf16 neighbours that the kernel's fp32 arithmetic may land on the
other side, both bf16 values are correct inputs to the quantisation; nowhere
else is there any freedom.  So every 16-element block must either equal the
oracle's bytes (8 code bytes and the E4M3 scale), or equal the oracle's
quantisation of the same block with some of its near-midpoint elements moved to
their other bf16 neighbour.  Nothing else passes: a wrong scale or code in any
other block fails, whatever fraction of the tensor it touches.

DELTA bounds the kernel's fp32 error relative to the exact value.  RMSNorm in
fp32 (per-thread sums of <= 40 squares, a tree over 128 threads, a correctly
rounded reciprocal square root, two multiplies) stays within ~2e-6 relative in
the worst case; SwiGLU (expf within 2 ulp, one add, one correctly rounded
division, one multiply) within ~1e-6.  DELTA = 2^-17 (7.6e-6) covers both.
"""
import numpy as np

DELTA = 2.0 ** -17


def bf16_of(y64: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 -> bf16 (round to nearest even), returned as fp64."""
    b = np.asarray(y64, np.float64).astype(np.float32).view(np.uint32)
    r = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def bf16_candidates(y64: np.ndarray, delta: float = DELTA):
    """(yb, nb): yb = the bf16 value the oracle takes; nb = its other bf16
    neighbour on the side of y64 where y64 lies within delta*|y64| of the
    midpoint between the two, else NaN."""
    y64 = np.asarray(y64, np.float64)
    yb = bf16_of(y64)
    bits = (yb.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    mag, sign = bits & 0x7FFF, bits & 0x8000
    up = np.abs(y64) > np.abs(yb)
    nmag = np.where(up, mag + 1, mag - 1)
    valid = nmag >= 0
    nbits = ((sign | np.clip(nmag, 0, 0x7FFF)) << 16).astype(np.uint32)
    nb = nbits.view(np.float32).astype(np.float64)
    mid = 0.5 * (yb + nb)
    amb = valid & (np.abs(y64 - mid) <= delta * np.abs(y64))
    return yb, np.where(amb, nb, np.nan)


def check_quant_bytes(oracle, y64, codes, scales, g, delta: float = DELTA, max_amb: int = 4):
    """Check a kernel's NVFP4 bytes (codes u8 [rows, n/2], scales u8 [rows, n/16])
    of bf16(y64) quantised with tensor scale g.  Returns (mismatching blocks,
    of them explained by near-midpoint elements); raises AssertionError on a
    block no correct bf16 input explains."""
    y64 = np.asarray(y64, np.float64)
    rows, n = y64.shape
    kb = n // 16
    yb, nb = bf16_candidates(y64, delta)
    oc, osc, _ = oracle.quantize(yb.astype(np.float32), g_in=g)
    cg = np.asarray(codes).reshape(rows, kb, 8)
    sg = np.asarray(scales).reshape(rows, kb)
    bad = (cg != oc.reshape(rows, kb, 8)).any(-1) | (sg != osc)
    idx = np.argwhere(bad)
    for r, b in idx:
        sl = slice(16 * b, 16 * b + 16)
        amb = np.flatnonzero(~np.isnan(nb[r, sl]))
        assert 0 < len(amb) <= max_amb, (
            f"block (row {r}, block {b}): kernel bytes differ from the oracle's and no element of the block "
            f"is within {delta:.1e} of a bf16 rounding midpoint ({len(amb)} near-midpoint elements)")
        cands = []
        for mask in range(1, 1 << len(amb)):
            v = yb[r, sl].copy()
            for j, e in enumerate(amb):
                if (mask >> j) & 1:
                    v[e] = nb[r, sl][e]
            cands.append(v)
        cc, cs, _ = oracle.quantize(np.array(cands, np.float32), g_in=g)
        ok = any(np.array_equal(cc[i], cg[r, b]) and cs[i, 0] == sg[r, b] for i in range(len(cands)))
        assert ok, f"block (row {r}, block {b}): kernel bytes match no correct bf16 rounding of the block"
    return len(idx), len(idx)
