"""Pins of the quantisation-prologue oracle (CPU): a hand-derived golden
case, the closed form of the scale, invariants, and per-head independence."""
import os

import numpy as np
import pytest

from oracle import quantize as oq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_half_even.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        k, v = line.split(":")
        vals[k.strip()] = [float(t) for t in v.split()]
    return vals


def test_golden_half_even():
    g = _golden()
    x = np.array(g["values"], dtype=np.float32).reshape(1, 1, 1, -1)
    codes, s = oq.quantize(x, per_head=True)
    assert codes.ravel().tolist() == [int(c) for c in g["codes"]]
    assert s.tolist() == g["scale"]


def test_scale_is_amax_over_127_and_max_maps_to_127():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 3, 5, 8)).astype(np.float32) * np.array([1, 10, 0.01], np.float32)[None, :, None, None]
    codes, s = oq.quantize(x, per_head=True)
    for h in range(3):
        amax = np.abs(x[:, h]).max()
        assert s[h] == np.float32(amax) / np.float32(127)
        i = np.unravel_index(np.abs(x[:, h]).argmax(), x[:, h].shape)
        assert abs(int(codes[:, h][i])) == 127
    assert np.abs(codes).max() <= 127


def test_reconstruction_error_is_half_a_step():
    rng = np.random.default_rng(4)
    x = (rng.standard_t(4, (2, 2, 16, 8)) * 3).astype(np.float32)
    codes, s = oq.quantize(x, per_head=False)
    err = np.abs(x.astype(np.float64) - codes.astype(np.float64) * float(s[0]))
    assert err.max() <= 0.5 * float(s[0]) * (1 + 1e-6)


def test_per_head_scales_are_independent():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 4, 8, 8)).astype(np.float32)
    c0, s0 = oq.quantize(x, per_head=True)
    y = x.copy()
    y[:, 2] *= 1000
    c1, s1 = oq.quantize(y, per_head=True)
    assert np.array_equal(np.delete(c0, 2, axis=1), np.delete(c1, 2, axis=1))
    assert np.array_equal(np.delete(s0, 2), np.delete(s1, 2))


def test_all_zero_tensor_has_unit_scale():
    codes, s = oq.quantize(np.zeros((1, 2, 3, 8), np.float32), per_head=True)
    assert s.tolist() == [1.0, 1.0] and not codes.any()


@pytest.mark.parametrize("per_head", [False, True])
def test_exact_rational_rounding_small_case(per_head):
    """code = nearest integer to x / s (ties to even), up to the single fp32
    rounding of the quotient: checked with exact rationals."""
    from fractions import Fraction
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((1, 2, 4, 8)) * 5).astype(np.float32)
    codes, s = oq.quantize(x, per_head)
    for idx in np.ndindex(x.shape):
        sh = s[idx[1]] if per_head else s[0]
        exact = Fraction(float(x[idx])) / Fraction(float(sh))
        assert abs(Fraction(int(codes[idx])) - exact) <= Fraction(1, 2) + Fraction(1, 10**5)
