"""Pins of the asymmetric quantisation oracle (``oracle.quantize.quantize_asym``:
u8 codes with a zero-point, the forum page "IntAttention：面向边缘设备的纯整数注意力推理加速方案",
section 动态量化策略) and planted mistakes that each must fail one.

The pins are functions of an implementation, so the mutants at the bottom
run them against planted-mistake restatements of the definition."""
import os

import numpy as np
import pytest

from oracle import quantize as oq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_zero_point.txt")
F32_MAX = np.finfo(np.float32).max


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, v = line.split(":")
        vals[key.strip()] = [float(t) for t in v.split()]
    return vals


def pin_golden(qa):
    g = _golden()
    for case in ("ties", "clamp", "positive", "recip", "odd"):
        x = np.array(g[case + "_values"], np.float32).reshape(1, 1, 1, -1)
        for per_head in (False, True):
            c, s, z = qa(x, per_head)
            assert c.ravel().tolist() == [int(t) for t in g[case + "_codes"]], case
            assert float(s[0]) == g[case + "_scale"][0], case
            assert int(z[0]) == int(g[case + "_zero_point"][0]), case


def _data(seed, shape=(2, 4, 37, 64), shift=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    if shift is not None:
        x += np.asarray(shift, np.float32).reshape(1, -1, 1, 1)
    return x.astype(np.float16).astype(np.float32)  # values an fp16 tensor holds


def pin_zero_is_the_zero_point(qa):
    """0 lies in every range, so the code of 0 is exactly z, and z in [0, 255]."""
    x = _data(1, shift=[3.0, -3.0, 0.0, 10.0])
    x[0, :, 0, 0] = 0.0
    c, s, z = qa(x, True)
    assert ((z >= 0) & (z <= 255)).all()
    assert np.array_equal(c[0, :, 0, 0].astype(np.int32), z)


def pin_reconstruction_within_half_step(qa):
    """|s (c - z) - x| <= s/2 (+ the float rounding of x * inv and of z), for
    every element of a head whose range is two-sided."""
    x = _data(2, shift=[1.0, -1.5, 0.0, 0.5])
    c, s, z = qa(x, True)
    for h in range(x.shape[1]):
        rec = float(s[h]) * (c[:, h].astype(np.float64) - int(z[h]))
        err = np.abs(rec - x[:, h].astype(np.float64)).max()
        assert err <= float(s[h]) * (1.0 + 1e-3), (h, err, float(s[h]))


def pin_extremes_use_the_whole_code_range(qa):
    """The head max maps to 255 (or 254 after a tie) and the head min to 0 (or 1)."""
    x = _data(3, shift=[0.3, -0.2, 2.0, -2.0])
    c, s, z = qa(x, True)
    for h in range(x.shape[1]):
        hmax, hmin = x[:, h].max(), x[:, h].min()
        if hmax > 0:
            assert c[:, h][x[:, h] == hmax].min() >= 254
        if hmin < 0:
            assert c[:, h][x[:, h] == hmin].max() <= 1


def pin_scale_closed_form(qa):
    """s = RN32((hi - lo) / 255) with the range widened to hold 0."""
    x = _data(4, shift=[4.0, -4.0, 0.0, 0.0])
    c, s, z = qa(x, True)
    for h in range(x.shape[1]):
        hi = max(float(x[:, h].max()), 0.0)
        lo = min(float(x[:, h].min()), 0.0)
        assert float(s[h]) == float(np.float32((hi - lo) / 255.0))
    # one-sided: the range still starts at 0, so z = 0 (all positive) or 255 (all negative)
    y = np.abs(_data(5, shape=(1, 2, 8, 64))) + np.float32(0.25)
    y[:, 1] *= -1
    _, s2, z2 = qa(y, True)
    assert z2.tolist() == [0, 255]


def pin_per_head_independent(qa):
    x = _data(6, shift=[0.0, 5.0, -5.0, 1.0])
    c, s, z = qa(x, True)
    for h in range(x.shape[1]):
        ch, sh, zh = qa(x[:, h:h + 1], False)
        assert np.array_equal(ch, c[:, h:h + 1]) and float(sh[0]) == float(s[h]) and int(zh[0]) == int(z[h])


def pin_per_tensor_range_spans_heads_and_batch(qa):
    x = _data(7, shift=[0.0, 5.0, -5.0, 1.0])
    c, s, z = qa(x, False)
    hi, lo = float(x.max()), float(x.min())
    assert float(s[0]) == float(np.float32((hi - lo) / 255.0))
    x2 = x.copy()
    x2[1, 2, 3, 4] = np.float32(40.0)  # a new maximum in batch entry 1 changes every head's codes
    c2, s2, z2 = qa(x2, False)
    assert float(s2[0]) > float(s[0])


def pin_all_zero_and_empty(qa):
    x = np.zeros((1, 2, 4, 64), np.float32)
    c, s, z = qa(x, True)
    assert not c.any() and s.tolist() == [1.0, 1.0] and z.tolist() == [0, 0]
    c, s, z = qa(np.zeros((0, 2, 4, 64), np.float32), True)
    assert c.size == 0 and s.tolist() == [1.0, 1.0] and z.tolist() == [0, 0]


def pin_exact_rational_rounding(qa):
    """Every code equals the definition evaluated with exact rationals of the
    fp32 values (the product rounded to fp32 first, ties to even)."""
    from fractions import Fraction
    x = _data(8, shape=(1, 1, 16, 16), shift=[0.7])
    c, s, z = qa(x, False)
    hi, lo = max(float(x.max()), 0.0), min(float(x.min()), 0.0)
    inv = np.float32(min(255.0 / (hi - lo), float(F32_MAX)))
    zz = int(np.clip(np.rint(np.float32(-lo) * inv), 0, 255))
    for xv, cv in zip(x.ravel(), c.ravel()):
        p = Fraction(float(np.float32(xv) * inv))  # RN32 of the exact product
        r = round(p)  # Fraction.__round__ is half-even
        assert int(cv) == min(max(r + zz, 0), 255)


PINS = [pin_golden, pin_zero_is_the_zero_point, pin_reconstruction_within_half_step,
        pin_extremes_use_the_whole_code_range, pin_scale_closed_form, pin_per_head_independent,
        pin_per_tensor_range_spans_heads_and_batch, pin_all_zero_and_empty, pin_exact_rational_rounding]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oq.quantize_asym)


# ------------------------------------------------------------- planted mistakes

def make_quantize_asym(range_without_zero=False, z_floor=False, z_before_rint=False, levels=255,
                       width_f32=False, no_clamp=False, z_from_hi=False, division=False):
    def qa(x, per_head):
        x = np.asarray(x, dtype=np.float32)
        B, H, L, d = x.shape
        n = H if per_head else 1
        axes = (0, 2, 3) if per_head else None
        if x.size:
            hi = np.asarray(x.max(axis=axes), np.float32).reshape(n)
            lo = np.asarray(x.min(axis=axes), np.float32).reshape(n)
        else:
            hi = lo = np.zeros(n, np.float32)
        if not range_without_zero:
            hi = np.maximum(hi, np.float32(0))
            lo = np.minimum(lo, np.float32(0))
        w = (hi - lo).astype(np.float64) if width_f32 else hi.astype(np.float64) - lo.astype(np.float64)
        s = np.ones(n, np.float32)
        inv = np.ones(n, np.float32)
        nz = w != 0
        s[nz] = (w[nz] / float(levels)).astype(np.float32)
        inv[nz] = np.minimum(float(levels) / w[nz], float(F32_MAX)).astype(np.float32)
        zr = (np.float32(levels) - hi * inv) if z_from_hi else (-lo) * inv
        z = np.floor(zr) if z_floor else np.rint(zr)
        z = np.clip(z, 0, 255).astype(np.int32)
        pi = inv if per_head else np.repeat(inv, H)
        pz = z if per_head else np.repeat(z, H)
        ps = s if per_head else np.repeat(s, H)
        with np.errstate(divide="ignore", invalid="ignore"):
            if division:
                prod = x / ps[None, :, None, None]
            else:
                prod = x * pi[None, :, None, None].astype(np.float32)
        if z_before_rint:
            q = np.rint(prod.astype(np.float32) + pz[None, :, None, None].astype(np.float32))
        else:
            q = np.rint(prod) + pz[None, :, None, None]
        q = q if no_clamp else np.clip(q, 0, 255)
        return (q.astype(np.int64) & 255).astype(np.uint8), s, z
    return qa


MUTANTS = {
    "range_without_zero": dict(range_without_zero=True),
    "zero_point_floored": dict(z_floor=True),
    "zero_point_added_before_rounding": dict(z_before_rint=True),
    "256_levels": dict(levels=256),
    "no_clamp_at_255": dict(no_clamp=True),
    "zero_point_from_the_top": dict(z_from_hi=True),
    "division_by_scale": dict(division=True),
}


def test_restatement_without_mistakes_equals_the_oracle():
    qa = make_quantize_asym()
    for seed, shift in ((20, [0.5, -1.0, 2.0, 0.0]), (21, [5.0, -5.0, 0.1, -0.1])):
        x = _data(seed, shift=shift)
        for ph in (False, True):
            a, b = qa(x, ph), oq.quantize_asym(x, ph)
            assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
    for pin in PINS:
        pin(qa)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    qa = make_quantize_asym(**MUTANTS[name])
    caught = []
    for pin in PINS:
        try:
            pin(qa)
        except Exception:  # noqa: BLE001 - any failing pin catches it
            caught.append(pin.__name__)
    assert caught, f"no pin catches {name}"
