"""Planted mistakes: each mutant copy of the oracle must fail at least one pin.

A mutant is the oracle source with one plausible slip (a dropped rounding
term, a wrong sign, a transposed operand, an off-by-one), compiled into a
temporary library on the CPU.  The pins are re-run against it; a mutant that
passes every pin would mean the pins cannot see that kind of mistake.
"""
import importlib.util
import os
import shutil
import subprocess

import numpy as np
import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "intattn_oracle.c")

MUTANTS = {
    "index_rounding_dropped": ("int64_t t = g * (int64_t)M + ((int64_t)1 << (s - 1));",
                               "int64_t t = g * (int64_t)M;"),
    "gap_sign_flipped": ("lut[oracle_index((int64_t)m - S[j], M, s, D)];\n    uint64_t R",
                         "lut[oracle_index((int64_t)S[j] - m, M, s, D)];\n    uint64_t R"),
    "lut_tail_not_zeroed": ("lut[31] = 0;", "lut[31] = (int32_t)llround(32768.0 * exp(-c));"),
    "lut_spacing_off_by_one": ("exp(-((double)i * c) / 31.0)", "exp(-((double)i * c) / 32.0)"),
    "reciprocal_rounding_dropped": ("((255ULL << 32) + (uint64_t)(Z / 2)) / (uint64_t)Z",
                                    "((255ULL << 32)) / (uint64_t)Z"),
    "prob_rounding_dropped": ("((E * R + (1ULL << 31)) >> 32)", "((E * R) >> 32)"),
    "normalise_to_256": ("(255ULL << 32)", "(256ULL << 32)"),
    "requant_rounding_dropped": ("(int64_t)acc * (int64_t)Mo + ((int64_t)1 << (so - 1));",
                                 "(int64_t)acc * (int64_t)Mo;"),
    "v_transposed": ("(int32_t)v[(size_t)j * d + t]", "(int32_t)v[(size_t)t * d + j]"),
    "k_index_uses_query_row": ("(int32_t)k[(size_t)j * d + t]", "(int32_t)k[(size_t)t]"),
    "no_sqrt_d": ("(s_q * s_k) / sqrt((double)d)", "(s_q * s_k)"),
    "causal_off_by_one": ("n = (int)(last + 1 < J->Lk ? last + 1 : J->Lk);",
                          "n = (int)(last < J->Lk ? last : J->Lk);"),
    "clip_missing": ("int64_t g = gap < (int64_t)D ? gap : (int64_t)D;",
                     "int64_t g = gap;"),
    "max_taken_as_first": ("if (S[j] > m) m = S[j];", "if (0) m = S[j];"),
    "requant_no_clamp": ("if (y > 127) y = 127;", "if (y > 300) y = 127;"),
}

PIN_TESTS = [
    ("test_lut_endpoints_monotone_and_rounding", {"c": 8.0}),
    ("test_lut_ratio_is_geometric", {}),
    ("test_index_multiplier_approximates_real_ratio", dict(zip("sq sk d c".split(), pins.SCALE_CASES[0]))),
    ("test_index_is_rounded_scaled_gap", dict(zip("sq sk d c".split(), pins.SCALE_CASES[3]))),
    ("test_requant_golden_half", {}),
    ("test_scores_match_integer_matmul", {}),
    ("test_uniform_rows_golden", {}),
    ("test_single_dominant_key", {}),
    ("test_probabilities_track_real_ratio", {}),
    ("test_brute_force_against_fp_attention", {"L": 32, "d": 64, "causal": False, "c": 8.0}),
    ("test_brute_force_against_fp_attention", {"L": 24, "d": 64, "causal": True, "c": 6.0}),
    ("test_single_key_reproduces_v", {}),
    ("test_causal_rows_ignore_masked_keys", {}),
    ("test_linearity_in_v_before_requant", {}),
]


def _load_mutant(tmp_path, name, before, after):
    src = open(SRC).read()
    assert src.count(before) >= 1, f"mutation anchor for {name} not found"
    mdir = tmp_path / name
    mdir.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), mdir / "__init__.py")
    (mdir / "intattn_oracle.c").write_text(src.replace(before, after, 1))
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", mdir / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _run_pins(mod):
    caught = []
    for fn, kw in PIN_TESTS:
        try:
            getattr(pins, fn)(mod, **kw)
        except Exception:  # noqa: BLE001 - any failing pin catches the mutant
            caught.append(fn)
    return caught


_CHILD = """
import sys, pathlib
sys.path[:0] = [{tests!r}, {root!r}]
import test_oracle_mutants as tm
mod = tm._load_mutant(pathlib.Path({tmp!r}), {name!r}, *tm.MUTANTS[{name!r}])
print("LOADED", flush=True)
print("CAUGHT", ",".join(tm._run_pins(mod)))
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    """Run in a child process: an out-of-range mutant may crash, which also
    counts as caught."""
    import sys
    assert open(SRC).read().count(MUTANTS[name][0]) >= 1, "mutation anchor not found"
    code = _CHILD.format(tests=os.path.dirname(os.path.abspath(__file__)), root=ROOT,
                         tmp=str(tmp_path), name=name)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert "LOADED" in r.stdout, r.stderr[-2000:]
    if r.returncode != 0:
        return  # crashed or raised while running the pins: the mistake is visible
    line = [x for x in r.stdout.splitlines() if x.startswith("CAUGHT")][-1]
    assert line.strip() != "CAUGHT", f"no pin catches mutant {name}"


def test_unmutated_copy_passes_every_pin(tmp_path):
    mod = _load_mutant(tmp_path, "identity", "#include <math.h>", "#include <math.h>")
    assert _run_pins(mod) == []
