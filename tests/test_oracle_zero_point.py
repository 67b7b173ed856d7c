"""Pins of the oracle's zero-point path (K and V as u8 codes with zero-points,
the forum page "IntAttention：面向边缘设备的纯整数注意力推理加速方案", section
动态量化策略: a dynamic scale and zero-point per layer).

A u8 code c with zero-point z stands for the integer c - z, so re-expressing
int8 codes x as x + z with zero-point z must leave every output byte as it
was; de-quantised, the output must track fp64 attention on real values
s (c - z).  Planted mistakes in the zero-point path must each fail a pin.
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest

from test_oracle_pins import _fp_attention

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "intattn_oracle.c")


def _case(rng, B, H, Lq, Lk, d, lo=-128, hi=127):
    q = rng.integers(-128, 128, (B, H, Lq, d)).astype(np.int8)
    k = rng.integers(lo, hi + 1, (B, H, Lk, d)).astype(np.int8)
    v = rng.integers(lo, hi + 1, (B, H, Lk, d)).astype(np.int8)
    return q, k, v


def _shift(x, z, per_head):
    """int8 codes x re-expressed as u8 codes x + z (z per head or one)."""
    z = np.asarray(z, dtype=np.int32)
    zz = z.reshape(1, -1, 1, 1) if per_head else z.reshape(1, 1, 1, 1)
    u = x.astype(np.int32) + zz
    assert u.min() >= 0 and u.max() <= 255
    return u.astype(np.uint8)


SCALES = dict(s_q=np.float32(0.02), s_k=np.float32(0.03), s_v=np.float32(0.05), s_o=np.float32(0.01))


@pytest.mark.parametrize("which", ["k", "v", "kv"])
@pytest.mark.parametrize("causal", [False, True])
def test_reexpressed_codes_give_the_same_bytes_per_tensor(oracle_mod, which, causal):
    rng = np.random.default_rng(11 + len(which) + causal)
    q, k, v = _case(rng, 2, 3, 20, 33, 64)
    base = oracle_mod.forward(q, k, v, False, *SCALES.values(), causal, 8.0)
    zk = 128 if "k" in which else None
    zv = 128 if "v" in which else None
    kk = _shift(k, 128, False) if zk is not None else k
    vv = _shift(v, 128, False) if zv is not None else v
    got = oracle_mod.forward(q, kk, vv, False, *SCALES.values(), causal, 8.0, z_k=zk, z_v=zv)
    assert np.array_equal(got, base)


def test_reexpressed_codes_give_the_same_bytes_per_head(oracle_mod):
    """Different zero-points per head: a wrong head index shows."""
    rng = np.random.default_rng(12)
    H = 4
    q, k, v = _case(rng, 2, H, 17, 40, 64, lo=-100, hi=55)
    sq = np.array([0.02, 0.03, 0.01, 0.05], np.float32)
    sk = np.array([0.03, 0.01, 0.02, 0.02], np.float32)
    sv = np.array([0.05, 0.02, 0.04, 0.03], np.float32)
    so = np.array([0.01, 0.005, 0.02, 0.01], np.float32)
    base = oracle_mod.forward(q, k, v, True, sq, sk, sv, so, True, 8.0)
    zk = np.array([100, 137, 200, 150], np.int32)
    zv = np.array([190, 100, 121, 173], np.int32)
    got = oracle_mod.forward(q, _shift(k, zk, True), _shift(v, zv, True), True, sq, sk, sv, so, True, 8.0,
                             z_k=zk, z_v=zv)
    assert np.array_equal(got, base)


def test_reexpressed_decode(oracle_mod):
    rng = np.random.default_rng(13)
    B, H, Lmax, d, Lk = 3, 2, 50, 128, 41
    q = rng.integers(-128, 128, (B, H, 1, d)).astype(np.int8)
    kc = rng.integers(-100, 56, (B, H, Lmax, d)).astype(np.int8)
    vc = rng.integers(-100, 56, (B, H, Lmax, d)).astype(np.int8)
    base = oracle_mod.decode(q, kc, vc, False, *SCALES.values(), Lk, 8.0)
    got = oracle_mod.decode(q, _shift(kc, 100, False), _shift(vc, 199, False), False, *SCALES.values(), Lk, 8.0,
                            z_k=100, z_v=199)
    assert np.array_equal(got, base)
    # a cache row beyond Lk does not matter
    vc2 = _shift(vc, 199, False)
    vc2[:, :, Lk:] = 255
    got2 = oracle_mod.decode(q, _shift(kc, 100, False), vc2, False, *SCALES.values(), Lk, 8.0, z_k=100, z_v=199)
    assert np.array_equal(got2, base)


def _asym_quant(x):
    """Real values -> u8 codes and a zero-point (a plain asymmetric rule, only
    to make test inputs: the pin below compares with real-valued attention)."""
    lo, hi = min(float(x.min()), 0.0), max(float(x.max()), 0.0)
    s = np.float32((hi - lo) / 255.0)
    z = int(np.clip(np.rint(-lo / float(s)), 0, 255))
    u = np.clip(np.rint(x / np.float64(s)) + z, 0, 255).astype(np.uint8)
    return u, s, z


@pytest.mark.parametrize("L,d,causal,c", [(16, 64, False, 8.0), (24, 64, True, 6.0), (32, 128, False, 10.0)])
def test_brute_force_against_fp_attention_with_zero_points(oracle_mod, L, d, causal, c):
    """K and V one-sided (shifted away from 0), so their zero-points are far
    from 128: de-quantised output vs fp64 softmax attention on the real
    values s (c - z): cosine >= 0.995, max-abs <= 0.05 max|V|."""
    rng = np.random.default_rng(200 + L + d)
    B, H = 2, 2
    q = rng.standard_normal((B, H, L, d)).astype(np.float32)
    kx = (rng.standard_normal((B, H, L, d)) + 2.5).astype(np.float32)
    vx = (rng.standard_normal((B, H, L, d)) - 2.0).astype(np.float32)
    sq = np.float32(np.abs(q).max() / 127.0)
    qc = np.clip(np.rint(q / np.float64(sq)), -127, 127).astype(np.int8)
    ku, sk, zk = _asym_quant(kx)
    vu, sv, zv = _asym_quant(vx)
    assert zk < 64 and zv > 160  # genuinely asymmetric ranges
    kr = (ku.astype(np.float64) - zk)  # the integers the codes stand for
    vr = (vu.astype(np.float64) - zv)
    ref = _fp_attention(qc, kr, vr, float(sq), float(sk), float(sv), causal)
    so = np.float32(np.abs(ref).max() / 127.0)
    out = oracle_mod.forward(qc, ku, vu, False, sq, sk, sv, so, causal, c, z_k=zk, z_v=zv)
    got = out.astype(np.float64) * float(so)
    cos = float((got * ref).sum() / (np.linalg.norm(got) * np.linalg.norm(ref)))
    vmax = float(np.abs(vr).max()) * float(sv)
    assert cos >= 0.995, cos
    assert np.abs(got - ref).max() <= 0.05 * vmax


def test_zero_point_out_of_range_is_rejected(oracle_mod):
    rng = np.random.default_rng(14)
    q, k, v = _case(rng, 1, 1, 4, 4, 64, lo=0, hi=100)
    for bad in (256, -1):
        with pytest.raises(Exception):
            oracle_mod.forward(q, k.astype(np.uint8), v, False, *SCALES.values(), False, 8.0, z_k=bad)


def test_row_probabilities_sum_to_at_most_510(oracle_mod):
    """Sum_j P_j <= 510 for every row (each key with P >= 1 has E/Z >= (1/2 -
    2^-18)/255, so at most 510 of them, each rounded up by at most 1/2):
    uniform rows of n keys reach 510 at n = 510 and fall to 0 at n = 511."""
    M, s, D = oracle_mod.index_params(0.05, 0.05, 64, 8.0)
    lut = oracle_mod.lut(8.0)
    for n, want in ((509, 509), (510, 510), (511, 0)):
        P = oracle_mod.index_softmax(np.zeros(n, np.int32), M, s, D, lut)[0]
        assert int(P.astype(np.int64).sum()) == want
    rng = np.random.default_rng(15)
    worst = 0
    for _ in range(300):
        n = int(rng.integers(1, 2000))
        S = rng.integers(-3000, 1, n).astype(np.int32)
        P = oracle_mod.index_softmax(S, M, s, D, lut)[0]
        worst = max(worst, int(P.astype(np.int64).sum()))
    assert worst <= 510


# ------------------------------------------------------------- planted mistakes

MUTANTS = {
    "v_zero_point_dropped": ("acc[t] += (int32_t)P[j] * (code_at(vz, v_u8, (size_t)j * d + t) - zv);",
                             "acc[t] += (int32_t)P[j] * (code_at(vz, v_u8, (size_t)j * d + t));"),
    "v_zero_point_added": ("(code_at(vz, v_u8, (size_t)j * d + t) - zv)", "(code_at(vz, v_u8, (size_t)j * d + t) + zv)"),
    "v_code_read_signed": ("code_at(vz, v_u8, (size_t)j * d + t)", "code_at(vz, 0, (size_t)j * d + t)"),
    "k_code_read_signed": ("code_at(kz, k_u8, (size_t)j * d + t)", "code_at(kz, 0, (size_t)j * d + t)"),
    "zero_point_of_head_0": ("J->zv ? J->zv[h] : 0", "J->zv ? J->zv[0] : 0"),
}

_CHILD = """
import sys, pathlib
sys.path[:0] = [{tests!r}, {root!r}]
import numpy as np
import test_oracle_mutants as tm
import test_oracle_zero_point as tz
mod = tm._load_mutant(pathlib.Path({tmp!r}), {name!r}, *tz.MUTANTS[{name!r}])
print("LOADED", flush=True)
caught = []
for fn, args in [("test_reexpressed_codes_give_the_same_bytes_per_tensor", ("kv", False)),
                 ("test_reexpressed_codes_give_the_same_bytes_per_head", ()),
                 ("test_reexpressed_decode", ())]:
    try:
        getattr(tz, fn)(mod, *args)
    except Exception:
        caught.append(fn)
print("CAUGHT", ",".join(caught))
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_zero_point_mutant_is_caught(tmp_path, name):
    assert open(SRC).read().count(MUTANTS[name][0]) >= 1, "mutation anchor not found"
    code = _CHILD.format(tests=os.path.dirname(os.path.abspath(__file__)), root=ROOT, tmp=str(tmp_path),
                         name=name)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert "LOADED" in r.stdout, r.stderr[-2000:]
    if r.returncode != 0:
        return
    line = [x for x in r.stdout.splitlines() if x.startswith("CAUGHT")][-1]
    assert line.strip() != "CAUGHT", f"no pin catches mutant {name}"
