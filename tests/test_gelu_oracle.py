"""Pins of the integer-GELU oracle (``oracle/gelu.py``) to facts outside it:
a hand-derived case, the normal CDF from another implementation, the
symmetry Phi(-t) = 1 - Phi(t), index invariants, the saturated ends, and an
error bound against the real GELU derived from the table spacing.

Each check is a function of the oracle module so that
``test_gelu_mutants`` can re-run it against planted mistakes."""
import math
import os

import numpy as np
import pytest

from oracle import gelu as oracle_gelu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "gelu_small.txt")
CODES = np.arange(-128, 128, dtype=np.int64)
# (s_x, s_y, c): activation-like input scales, output scale >= input scale
# (GELU(x) <= max(x, 0), so no clamp binds), gate ranges 3..6
PARAM_CASES = [(0.125, 0.125, 3.875), (0.04, 0.04, 4.0), (5.0 / 127, 6.0 / 127, 3.0),
               (0.3, 0.35, 6.0), (0.01, 0.02, 4.5)]
PHI_MAX = 1.0 / math.sqrt(2.0 * math.pi)  # max of the normal density


def check_golden(g):
    p = g.gelu_params(0.125, 0.125, 3.875)
    assert p[0] == 1 << 24 and p[1] == 25 and p[3] == 1 << 30 and p[4] == 45
    rows = [list(map(int, ln.split())) for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 10
    for q, idx, G, out in rows:
        assert int(g.gelu_index(q, p[0], p[1])) == idx, q
        assert p[2][idx] == G, q
        assert int(g.gelu_codes(np.array([q]), p)[0]) == out, q


def check_table_is_rounded_normal_cdf(g, c):
    from scipy.special import ndtr
    G = g.gelu_params(0.05, 0.05, c)[2]
    assert G[0] == 0 and G[31] == 32768
    for i in range(1, 31):
        v = 32768.0 * float(ndtr(((2 * i - 31) * float(np.float32(c))) / 31.0))
        if abs(v - math.floor(v) - 0.5) < 1e-6:
            continue  # too close to a rounding tie to judge by another implementation
        assert G[i] == math.floor(v + 0.5), (i, G[i], v)


def check_table_symmetry(g, c):
    G = g.gelu_params(0.05, 0.05, c)[2]
    for i in range(1, 31):
        assert G[i] + G[31 - i] in (32767, 32768, 32769), i
    assert all(G[i] <= G[i + 1] for i in range(31))


def check_index_invariants(g, s_x, c):
    M, s, *_ = g.gelu_params(s_x, s_x, c)
    idx = g.gelu_index(CODES, M, s)
    assert idx[128] == 16  # q = 0
    assert np.all(np.diff(idx) >= 0) and idx.min() >= 0 and idx.max() <= 31
    # floor(qM/2^s) + floor(-qM/2^s) = -1 unless qM/2^s is an integer
    for q in range(1, 128):
        a = int(g.gelu_index(q, M, s)) - 16
        b = int(g.gelu_index(-q, M, s)) - 16
        if -16 < b and a < 15:  # neither end clamped
            exact = (q * M) % (1 << s) == 0
            assert a + b == (0 if exact else -1), q
    # the index is the table point nearest x = s_x q (round half up), within
    # the multiplier's quantisation of r = s_x 31 / (2c)
    r = (float(np.float32(s_x)) * 31.0) / (2.0 * float(np.float32(c)))
    for q in CODES:
        i = int(g.gelu_index(int(q), M, s))
        if 0 < i < 31:
            assert abs(i - (q * r + 15.5)) <= 0.5 + 128 * abs(M / 2.0 ** s - r) + 1e-12, q


def check_error_bound(g, s_x, s_y, c):
    """|GELU(s_x q) - s_y out(q)| <= |x| e_gate + s_y (1/2 + 1e-6) for every code."""
    p = g.gelu_params(s_x, s_y, c)
    M, s = p[0], p[1]
    sx, sy, cc = (float(np.float32(v)) for v in (s_x, s_y, c))
    r = (sx * 31.0) / (2.0 * cc)
    drift = 128 * abs(M / 2.0 ** s - r) * (2.0 * cc / 31.0)  # index error, in x units
    half = cc / 31.0  # half the table spacing
    interior = PHI_MAX * (half + drift) + 0.5 / 32768
    ends = 0.5 * math.erfc((cc - half - drift) / math.sqrt(2.0))  # 1 - Phi(c - half - drift)
    e_gate = max(interior, ends)
    out = g.gelu_codes(CODES, p).astype(np.int64)
    for q, o in zip(CODES, out):
        x = sx * int(q)
        bound = abs(x) * (e_gate + 1e-6) + sy * (0.5 + 1e-6)
        assert abs(g.gelu_real(x) - sy * int(o)) <= bound, (int(q), int(o), g.gelu_real(x) / sy)


def check_saturated_ends(g, s_x, c):
    """s_y = s_x: gate 1 passes the code through, gate 0 gives 0, 0 -> 0."""
    p = g.gelu_params(s_x, s_x, c)
    idx = g.gelu_index(CODES, p[0], p[1])
    out = g.gelu_codes(CODES, p).astype(np.int64)
    assert out[128] == 0
    assert np.array_equal(out[idx == 31], CODES[idx == 31])
    assert not out[idx == 0].any()
    if s_x * 127 > c * 32 / 31:  # the codes reach both ends of the table
        assert (idx == 31).any() and (idx == 0).any()


def check_requant_multiplier(g, s_x, s_y, c):
    _, _, _, Mo, so = g.gelu_params(s_x, s_y, c)
    m = float(np.float32(s_x)) / (32768.0 * float(np.float32(s_y)))
    assert (1 << 30) <= Mo < (1 << 31) and 1 <= so <= 62
    assert abs(Mo / 2.0 ** so - m) <= m * 2.0 ** -30


def check_clamp(g):
    """s_y = s_x / 2 doubles every code, so the clamp to +-127 binds."""
    p = g.gelu_params(0.125, 0.0625, 3.875)
    out = g.gelu_codes(CODES, p).astype(np.int64)
    assert out.max() == 127 and out.min() >= -127
    assert out[128 + 127] == 127 and out[128 + 64] == 127 and out[128 + 40] == 80


def check_llround(g):
    assert [g.llround(v) for v in (0.5, 1.5, 2.5, -0.5, -2.5, 0.49999999999999994, 2.0 ** 52 + 1)] == \
        [1, 2, 3, -1, -3, 0, 2 ** 52 + 1]


def test_golden_small():
    check_golden(oracle_gelu)


@pytest.mark.parametrize("c", [3.0, 3.875, 4.0, 6.0])
def test_table_is_rounded_normal_cdf(c):
    check_table_is_rounded_normal_cdf(oracle_gelu, c)


@pytest.mark.parametrize("c", [3.0, 4.0, 6.0])
def test_table_symmetry(c):
    check_table_symmetry(oracle_gelu, c)


@pytest.mark.parametrize("case", PARAM_CASES)
def test_index_invariants(case):
    check_index_invariants(oracle_gelu, case[0], case[2])


@pytest.mark.parametrize("case", PARAM_CASES)
def test_error_bound_against_real_gelu(case):
    check_error_bound(oracle_gelu, *case)


@pytest.mark.parametrize("case", PARAM_CASES)
def test_saturated_ends(case):
    check_saturated_ends(oracle_gelu, case[0], case[2])


@pytest.mark.parametrize("case", PARAM_CASES)
def test_requant_multiplier(case):
    check_requant_multiplier(oracle_gelu, *case)


@pytest.mark.parametrize("args", [(0.0, 0.1, 4.0), (0.1, -1.0, 4.0), (0.1, 0.1, 0.0), (float("inf"), 0.1, 4.0),
                                  (0.1, 0.1, float("nan")), (1e-12, 0.1, 1e6), (1e-10, 1e3, 4.0)])
def test_param_range(args):
    with pytest.raises(oracle_gelu.ParamRange):
        oracle_gelu.gelu_params(*args)


def test_clamp_binds():
    check_clamp(oracle_gelu)


def test_llround_halves_away_from_zero():
    check_llround(oracle_gelu)


def run_all_checks(g):
    """Every pin above against module g (used by the mutant tests)."""
    check_golden(g)
    check_llround(g)
    check_clamp(g)
    for c in (3.0, 3.875, 4.0, 6.0):
        check_table_is_rounded_normal_cdf(g, c)
        check_table_symmetry(g, c)
    for case in PARAM_CASES:
        check_index_invariants(g, case[0], case[2])
        check_error_bound(g, *case)
        check_saturated_ends(g, case[0], case[2])
        check_requant_multiplier(g, *case)
