"""CPU checks of two pieces of arithmetic the prefill kernels use in place of
the definition's integer steps (the GPU parity tests check them end to end;
these check every input of the ranges the kernels meet).

1. LUT index on the FP32 pipe.  For a row max m and score S the kernels form
   the float X = 2^23 + g (g = m - S, 0 <= g <= 2^22) from bit patterns, then
       y = fma.rz.sat(X, M 2^-(s+5), (3/2 - 2^23 M 2^-s) / 32)
       t = fma.rz(y, 32, 2^23)
   and read k = bits(t) - 0x4B000000.  The definition's index is
   idx = (min(g, D) M + 2^(s-1)) >> s; the kernels need k == idx + 1 (a table
   row; 32 for every clipped gap).  Each fp32 fma is emulated exactly: the
   products and sums are exact in float64 (at most 49 significant bits), and
   rounding toward zero to fp32 is applied to that exact value.

2. Tile geometry by multiply and shift.  floor(n / d) for 0 <= n < 2^31 as
   (n * m) >> sh with m = ceil(2^(31 + l) / d), sh = 31 + l, l = ceil(log2 d)
   (Granlund and Montgomery's round-up reciprocal for 31-bit dividends).
"""
import random

import numpy as np
import pytest


def _rz32(x: np.ndarray) -> np.ndarray:
    """float64 values (exact) -> fp32 rounded toward zero."""
    r = x.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(x)
    r[over] = np.nextafter(r[over], np.float32(0))
    return r


def _sat01(y: np.ndarray) -> np.ndarray:
    return np.minimum(np.maximum(y, np.float32(0)), np.float32(1))


def _index_params(r: float):
    """M, s, D of the definition for a ratio r = alpha * 31 / c."""
    s = 26
    while s > 1 and round(r * 2 ** s) > 2 ** 24:
        s -= 1
    M = round(r * 2 ** s)
    if M < 1 or M > 2 ** 24 or M > 2 ** s:
        return None
    D = (61 * 2 ** (s - 1) + M - 1) // M
    return M, s, D


RATIOS = [1.0, 0.5, 1 - 2 ** -20, 0.75, 0.3, 1e-3, 3e-7, 0.0191, 0.137, 0.00042]


@pytest.mark.parametrize("r", RATIOS)
def test_fp32_index_code_equals_definition(r):
    p = _index_params(r)
    assert p is not None
    M, s, D = p
    assert s in (24, 25, 26)  # the kernels' constants are exact only for these shifts
    g = np.arange(0, 2 ** 22 + 1, dtype=np.int64)
    want = ((np.minimum(g, D) * M + 2 ** (s - 1)) >> s) + 1
    X = (2.0 ** 23 + g).astype(np.float64)
    Ms32 = M * 2.0 ** -(s + 5)
    c1 = (1.5 - M * 2.0 ** (23 - s)) / 32
    assert np.float64(np.float32(Ms32)) == Ms32 and np.float64(np.float32(c1)) == c1
    y = _sat01(_rz32(X * Ms32 + c1))   # the rounding happens before the clamp; both toward [0, 1]
    t = _rz32(y.astype(np.float64) * 32 + 2.0 ** 23)
    k = t.view(np.uint32).astype(np.int64) - 0x4B000000
    bad = np.nonzero(k != want)[0]
    assert bad.size == 0, f"r={r}: first gap {g[bad[0]]} gives code {k[bad[0]]}, want {want[bad[0]]}"


def _div_magic(d: int):
    l = 0
    while (1 << l) < d:
        l += 1
    k = 31 + l
    m = ((1 << k) + d - 1) // d
    assert m < 2 ** 32
    return m, k


def test_magic_division_small_divisors_exhaustive_edges():
    for d in range(1, 4097):
        m, sh = _div_magic(d)
        ns = {0, 1, d - 1, d, d + 1, 2 ** 31 - 1, 2 ** 31 - d, (2 ** 31 // d) * d, (2 ** 31 // d) * d - 1}
        for n in ns:
            if 0 <= n < 2 ** 31:
                assert (n * m) >> sh == n // d, (n, d)


def test_magic_division_random():
    rng = random.Random(5)
    for _ in range(20000):
        d = rng.choice([rng.randrange(1, 2 ** 16), rng.randrange(1, 2 ** 31), 2 ** rng.randrange(0, 31)])
        m, sh = _div_magic(d)
        for n in (rng.randrange(0, 2 ** 31), rng.randrange(0, 2 ** 31)):
            assert (n * m) >> sh == n // d, (n, d)
