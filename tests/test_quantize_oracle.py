"""Pins of the quantisation-prologue oracle (CPU): hand-derived golden cases
(ties at both roundings, a reciprocal scale that is not 1, the FLT_MAX cap),
the closed form of the scale, invariants, and per-head independence.

Every pin is a function of the quantise implementation it checks, so that
``test_quantize_mutants.py`` can run the same pins against planted mistakes.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import quantize as oq

GOLDEN_DIR = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN_DIR, name)):
        if line.startswith("#") or not line.strip():
            continue
        k, v = line.split(":")
        vals[k.strip()] = [float(t) for t in v.split()]
    return vals


def _one_head(values):
    return np.array(values, dtype=np.float32).reshape(1, 1, 1, -1)


# ------------------------------------------------------------------ pins

def pin_golden_half_even(quantize):
    """amax = 127: s = inv = 1, so the codes are rint of the values."""
    g = _golden("quantize_half_even.txt")
    codes, s = quantize(_one_head(g["values"]), True)
    assert codes.ravel().tolist() == [int(c) for c in g["codes"]]
    assert s.tolist() == g["scale"]


def pin_golden_reciprocal_tie(quantize):
    """inv != 1: the fp32 product x * inv lands on a tie at fp32 precision
    (rounds to 63.5), then rint's tie goes to 64."""
    g = _golden("quantize_reciprocal_tie.txt")
    for per_head in (True, False):
        codes, s = quantize(_one_head(g["tie_values"]), per_head)
        assert codes.ravel().tolist() == [int(c) for c in g["tie_codes"]]
        assert s.tolist() == g["tie_scale"]


def pin_golden_cap(quantize):
    """127 / amax above FLT_MAX: inv is capped, zeros stay 0."""
    g = _golden("quantize_reciprocal_tie.txt")
    codes, s = quantize(_one_head(g["cap_values"]), True)
    assert codes.ravel().tolist() == [int(c) for c in g["cap_codes"]]
    assert float(s[0]) == g["cap_scale_units_of_2^-149"][0] * 2.0 ** -149


def pin_scale_closed_form(quantize):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 3, 5, 8)).astype(np.float32) * np.array([1, 10, 0.01], np.float32)[None, :, None, None]
    codes, s = quantize(x, True)
    for h in range(3):
        amax = np.abs(x[:, h]).max()
        assert s[h] == np.float32(amax) / np.float32(127)
        i = np.unravel_index(np.abs(x[:, h]).argmax(), x[:, h].shape)
        assert abs(int(codes[:, h][i])) == 127
    assert np.abs(codes).max() <= 127


def pin_reconstruction_half_step(quantize):
    rng = np.random.default_rng(4)
    x = (rng.standard_t(4, (2, 2, 16, 8)) * 3).astype(np.float32)
    codes, s = quantize(x, False)
    err = np.abs(x.astype(np.float64) - codes.astype(np.float64) * float(s[0]))
    assert err.max() <= 0.5 * float(s[0]) * (1 + 1e-6)


def pin_per_head_independent(quantize):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, 4, 8, 8)).astype(np.float32)
    c0, s0 = quantize(x, True)
    y = x.copy()
    y[:, 2] *= 1000
    c1, s1 = quantize(y, True)
    assert np.array_equal(np.delete(c0, 2, axis=1), np.delete(c1, 2, axis=1))
    assert np.array_equal(np.delete(s0, 2), np.delete(s1, 2))


def pin_per_head_range_spans_batch(quantize):
    """A head's range is over all batch entries of that head, not per entry."""
    x = np.zeros((2, 1, 1, 8), np.float32)
    x[0, 0, 0, 0] = 2.0
    x[1, 0, 0, 0] = 1.0
    codes, s = quantize(x, True)
    assert int(codes[1, 0, 0, 0]) == 64  # 1.0 * RN32(127 / 2) = 63.5 -> 64
    assert int(codes[0, 0, 0, 0]) == 127


def pin_all_zero_unit_scale(quantize):
    codes, s = quantize(np.zeros((1, 2, 3, 8), np.float32), True)
    assert s.tolist() == [1.0, 1.0] and not codes.any()


def pin_exact_rational_rounding(quantize):
    """code = nearest integer to x / s (ties to even), up to the fp32
    roundings of inv and of the product: checked with exact rationals."""
    rng = np.random.default_rng(6)
    for per_head in (False, True):
        x = (rng.standard_normal((1, 2, 4, 8)) * 5).astype(np.float32)
        codes, s = quantize(x, per_head)
        for idx in np.ndindex(x.shape):
            sh = s[idx[1]] if per_head else s[0]
            exact = Fraction(float(x[idx])) / Fraction(float(sh))
            assert abs(Fraction(int(codes[idx])) - exact) <= Fraction(1, 2) + Fraction(1, 10**5)


PINS = [pin_golden_half_even, pin_golden_reciprocal_tie, pin_golden_cap, pin_scale_closed_form,
        pin_reconstruction_half_step, pin_per_head_independent, pin_per_head_range_spans_batch,
        pin_all_zero_unit_scale, pin_exact_rational_rounding]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oq.quantize)
