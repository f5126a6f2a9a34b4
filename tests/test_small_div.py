"""CPU proof of the GEMM kernel's division-free unit decomposition: for every
numerator 0 <= n < 2^22 and the divisors the launch plan can produce, the
binary32 product n * rn(1/d), truncated toward zero and corrected once by the
remainder, equals the integer quotient n // d.  The steps are replayed with
numpy binary32 arithmetic (IEEE round-to-nearest for 1/d; the product is
exact in binary64 and then truncated as the kernel's round-toward-zero
multiply does)."""
import numpy as np
import pytest

N_MAX = 1 << 22


def _replay(n, d):
    rcp = np.float32(1.0) / np.float32(d)                 # rn(1/d)
    prod = n.astype(np.float64) * np.float64(rcp)         # exact (24 x 24 bits)
    # round toward zero to binary32, then truncate to an integer
    p32 = prod.astype(np.float32)
    over = np.abs(p32.astype(np.float64)) > np.abs(prod)
    p32 = np.where(over, np.nextafter(p32, np.float32(0)), p32)
    q = np.trunc(p32).astype(np.int64)
    r = n - q * d
    q = np.where(r < 0, q - 1, np.where(r >= d, q + 1, q))
    return q


@pytest.mark.parametrize("d", list(range(1, 17)) + [24, 33, 48, 97, 176, 384, 1024, 4095])
def test_small_div_exact(d):
    n = np.arange(N_MAX, dtype=np.int64)
    assert np.array_equal(_replay(n, d), n // d)
