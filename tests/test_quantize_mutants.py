"""Planted mistakes in the quantisation-prologue oracle: each must be caught
by at least one pin of ``test_quantize_oracle.py``.

The mutants are built from one parametrised restatement of the oracle's
definition; with no mistake planted it must agree with ``oracle.quantize``
exactly, so each mutant differs from the oracle in the one planted step.
"""
import numpy as np
import pytest

from oracle import quantize as oq
from tests.test_quantize_oracle import PINS

F32_MAX = np.finfo(np.float32).max


def make_quantize(division=False, fused=False, no_cap=False, per_tensor_range=False,
                  per_entry_range=False, half_away=False, scale_inverted=False, clamp128=False,
                  scale_f64=False):
    def quantize(x, per_head):
        x = np.asarray(x, dtype=np.float32)
        B, H, L, d = x.shape
        ph = per_head and not per_tensor_range
        if ph:
            axes = (2, 3) if per_entry_range else (0, 2, 3)
            amax = np.abs(x).max(axis=axes) if x.size else np.zeros(H, np.float32)
        else:
            amax = np.array([np.abs(x).max() if x.size else 0.0], np.float32)
        amax = amax.astype(np.float32)
        with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
            if scale_f64:
                s = (amax.astype(np.float64) / 127.0).astype(np.float32)
            else:
                s = (amax / np.float32(127.0)).astype(np.float32)
            inv = np.float32(127.0) / np.where(amax == 0, np.float32(1), amax)
            if not no_cap:
                inv = np.minimum(inv, F32_MAX)
            inv = inv.astype(np.float32)
        s = np.where(amax == 0, np.float32(1), s).astype(np.float32)
        inv = np.where(amax == 0, np.float32(1), inv).astype(np.float32)
        if scale_inverted:
            s = inv.copy()
        if ph and per_entry_range:  # amax [B, H]
            sel_inv = inv[:, :, None, None]
            sel_s = s[:, :, None, None]
            s = s.max(axis=0)
        else:
            sel_inv = (inv if ph else np.repeat(inv, H))[None, :, None, None]
            sel_s = (s if ph else np.repeat(s, H))[None, :, None, None]
        with np.errstate(over="ignore", invalid="ignore"):
            if division:
                p = x / sel_s
            elif fused:
                p = x.astype(np.float64) * sel_inv.astype(np.float64)
            else:
                p = x * sel_inv
            q = np.floor(np.abs(p) + 0.5) * np.sign(p) if half_away else np.rint(p)
            lo = -128 if clamp128 else -127
            q = np.clip(np.nan_to_num(q, nan=-128.0), lo, 127)
        if per_head and per_tensor_range:
            out_s = np.repeat(s, H)  # one entry per head, all from the tensor's range
        elif ph:
            out_s = s
        else:
            out_s = s[:1]
        return q.astype(np.int8), out_s.astype(np.float32)
    return quantize


MUTANTS = {
    "division_by_scale": dict(division=True),
    "product_not_rounded_to_fp32": dict(fused=True),
    "reciprocal_not_capped": dict(no_cap=True),
    "per_tensor_range_for_heads": dict(per_tensor_range=True),
    "range_per_batch_entry": dict(per_entry_range=True),
    "ties_away_from_zero": dict(half_away=True),
    "scale_is_reciprocal": dict(scale_inverted=True),
}


def test_restatement_matches_oracle():
    rng = np.random.default_rng(11)
    q = make_quantize()
    for per_head in (False, True):
        for scale in (1.0, 1e-3, 300.0):
            x = (rng.standard_t(4, (2, 3, 7, 8)) * scale).astype(np.float32)
            c0, s0 = oq.quantize(x, per_head)
            c1, s1 = q(x, per_head)
            assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    for pin in PINS:
        pin(q)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    q = make_quantize(**MUTANTS[name])
    caught = []
    for pin in PINS:
        try:
            pin(q)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name!r} passes every pin"
