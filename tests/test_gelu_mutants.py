"""Planted mistakes in the integer-GELU oracle: each mutant copy of
``oracle/gelu.py`` (one plausible slip each) must fail at least one pin of
``test_gelu_oracle``."""
import os
import types

import pytest

import test_gelu_oracle as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "gelu.py")

MUTANTS = {
    "index_offset_off_by_one": ("np.clip(16 + ((q * M) >> s), 0, 31)", "np.clip(15 + ((q * M) >> s), 0, 31)"),
    "index_sign_flipped": ("np.clip(16 + ((q * M) >> s), 0, 31)", "np.clip(16 + ((-q * M) >> s), 0, 31)"),
    "index_range_not_halved": ("r = (s_x * 31.0) / (2.0 * c)", "r = (s_x * 31.0) / c"),
    "index_steps_32": ("r = (s_x * 31.0) / (2.0 * c)", "r = (s_x * 32.0) / (2.0 * c)"),
    "gate_mirrored": ("0.5 * math.erfc(-t / math.sqrt(2.0))", "0.5 * math.erfc(t / math.sqrt(2.0))"),
    "gate_spacing_32": ("t = ((2 * i - 31) * c) / 31.0", "t = ((2 * i - 31) * c) / 32.0"),
    "gate_not_centred": ("t = ((2 * i - 31) * c) / 31.0", "t = ((2 * i - 32) * c) / 31.0"),
    "gate_top_not_one": ("    G[31] = 32768\n", "    G[31] = 32767\n"),
    "gate_scale_2_14": ("G[i] = llround(32768.0 * (0.5 *", "G[i] = llround(16384.0 * (0.5 *"),
    "requant_rounding_dropped": ("out = (y * Mo + (1 << (so - 1))) >> so", "out = (y * Mo) >> so"),
    "requant_scales_swapped": ("m = s_x / (32768.0 * s_y)", "m = s_y / (32768.0 * s_x)"),
    "requant_table_scale_dropped": ("m = s_x / (32768.0 * s_y)", "m = s_x / s_y"),
    "clamp_too_wide": ("np.clip(out, -127, 127)", "np.clip(out, -128, 128)"),
    "gate_applied_to_index": ("y = q * np.asarray(G, dtype=np.int64)[gelu_index(q, M, s)]",
                              "y = gelu_index(q, M, s) * np.asarray(G, dtype=np.int64)[gelu_index(q, M, s)]"),
    "llround_half_even": ("return int(f) + (1 if x - f >= 0.5 else 0)", "return round(x)"),
}


def _mutant(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mod = types.ModuleType("gelu_mutant_" + name)
    exec(compile(src.replace(old, new), SRC + ":" + name, "exec"), mod.__dict__)
    return mod


def test_unmutated_oracle_passes_every_pin():
    pins.run_all_checks(_mutant_free())


def _mutant_free():
    mod = types.ModuleType("gelu_unmutated")
    exec(compile(open(SRC).read(), SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    g = _mutant(name)
    with pytest.raises(Exception):
        pins.run_all_checks(g)
