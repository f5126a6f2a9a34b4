"""The activation quantizer rounds x / sx without a division: q is rounded
from x * rcp(sx) and corrected with the exact remainder x - q * sx.  These
CPU checks cover the two facts that make its codes equal to rounding an IEEE
binary32 division (what the oracle does):

1. for FP16 x and FP16 sx > 0, rounding the binary32 quotient to the nearest
   integer (ties to even) equals rounding the exact quotient;
2. the procedure (rounding x * rcp(sx) with the 1.5 * 2^23 offset in one
   fused multiply-add, then correcting with the exact remainder), replayed
   here with numpy binary32 operations, returns the round-half-even of the
   exact quotient.
"""
import numpy as np


def _pairs(step):
    xs = np.arange(65536, dtype=np.uint16).view(np.float16)
    xs = xs[np.isfinite(xs)].astype(np.float32)
    ss = np.arange(1, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float32)
    return xs, ss[::step]


def test_binary32_quotient_rounds_like_exact_quotient():
    xs, ss = _pairs(97)
    for s in ss:
        q32 = np.rint(xs / np.float32(s))
        q64 = np.rint(xs.astype(np.float64) / np.float64(s))   # exact decision
        m = np.abs(q64) <= 130
        assert np.array_equal(q32[m], q64[m]), float(s)


def _remainder_rounding(x, s):
    """The kernel's steps with binary32 arithmetic."""
    magic = np.float64(12582912.0)                 # 1.5 * 2^23
    s = np.float32(s)
    rcp = np.float32(1.0) / s                      # correctly rounded reciprocal
    # fma(x, rcp, magic): x * rcp + magic is exact in binary64 here, one rounding
    t = (x.astype(np.float64) * np.float64(rcp) + magic).astype(np.float32)
    q = t.astype(np.float64) - magic               # exact integer
    # fma(-q, s, x): exact in binary64 and representable in binary32 here
    e = (x.astype(np.float64) - q * np.float64(s))
    assert np.array_equal(e.astype(np.float32).astype(np.float64), e)
    ae = np.abs(e)
    half = np.float64(s) / 2
    odd = (t.view(np.uint32) & 1) != 0             # parity of t is the parity of q
    move = (ae > half) | ((ae == half) & odd)
    return q + np.where(move, np.sign(e), 0)


def test_remainder_corrected_rounding_is_exact():
    xs, ss = _pairs(61)
    ties = 0
    for s in ss:
        q = _remainder_rounding(xs, s)
        q64 = np.rint(xs.astype(np.float64) / np.float64(s))
        m = np.abs(q64) <= 130
        assert np.array_equal(q[m], q64[m]), float(s)
        ties += int(np.sum(np.abs(xs.astype(np.float64) / np.float64(s) % 1 - 0.5)[m] == 0))
    assert ties > 1000          # the tie branch is exercised
