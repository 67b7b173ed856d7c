"""Pins of the adaptive clip threshold oracle (CPU): a hand-derived case,
invariances the rule must have, and a brute force restatement on tiny
inputs that shares nothing with the oracle's sort-based selection."""
import itertools
import os

import numpy as np
import pytest

from oracle import calibrate as oc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "calibrate_small.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, v = line.split(":")
        vals[key.strip()] = [float(t) for t in v.split()]
    return vals


def test_golden_gaps_and_threshold():
    g = _golden()
    q = np.array(g["q"], np.int8).reshape(1, 1, 4, 4)
    k = np.array(g["k"], np.int8).reshape(1, 1, 4, 4)
    assert oc.gaps(q, k, False, 2, 2)[0, 0] == g["G_keep2_stride2"][0]
    assert oc.gaps(q, k, False, 3, 1)[0, 0] == g["G_keep3_stride1"][0]
    assert oc.gaps(q, k, True, 3, 1)[0, 0] == g["G_keep3_stride1_causal"][0]
    c, G = oc.thresholds(q, k, True, [1.0], [1.0], False, 2, 2, 0.5, 20.0)
    assert float(c[0]) == g["c_keep2_stride2"][0]


def _brute_G(q, k, causal, keep, stride):
    """K-th largest by counting: the largest value t such that at least keep
    valid scores are >= t (or the row minimum when fewer are valid)."""
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    G = np.zeros((B, H), np.int64)
    for b, h in itertools.product(range(B), range(H)):
        for i in range(stride - 1, Lq, stride):
            n = min(Lk, i + Lk - Lq + 1) if causal else Lk
            s = [int(sum(int(q[b, h, i, t]) * int(k[b, h, j, t]) for t in range(d))) for j in range(n)]
            want = min(keep, n)
            kth = max(t for t in s if sum(1 for u in s if u >= t) >= want)
            G[b, h] = max(G[b, h], max(s) - kth)
    return G


@pytest.mark.parametrize("causal,keep,stride", [(False, 1, 1), (False, 3, 2), (True, 2, 1), (True, 5, 3)])
def test_gaps_brute_force(causal, keep, stride):
    rng = np.random.default_rng(keep * 10 + stride)
    q = rng.integers(-128, 128, (2, 2, 9, 8)).astype(np.int8)
    k = rng.integers(-128, 128, (2, 2, 11, 8)).astype(np.int8)
    assert np.array_equal(oc.gaps(q, k, causal, keep, stride), _brute_G(q, k, causal, keep, stride))


def test_keep_one_gives_zero_gap_and_c_min():
    rng = np.random.default_rng(7)
    q = rng.integers(-128, 128, (1, 2, 16, 8)).astype(np.int8)
    k = rng.integers(-128, 128, (1, 2, 16, 8)).astype(np.int8)
    assert not oc.gaps(q, k, False, 1, 1).any()
    c, _ = oc.thresholds(q, k, True, [0.1, 0.1], [0.1, 0.1], False, 1, 1, 0.75, 20.0)
    assert c.tolist() == [0.75, 0.75]


def test_gap_grows_with_keep_and_key_order_does_not_matter():
    rng = np.random.default_rng(8)
    q = rng.integers(-128, 128, (1, 1, 20, 16)).astype(np.int8)
    k = rng.integers(-128, 128, (1, 1, 30, 16)).astype(np.int8)
    prev = -1
    for keep in (1, 2, 4, 8, 30, 40):
        G = int(oc.gaps(q, k, False, keep, 1)[0, 0])
        assert G >= prev
        prev = G
    perm = rng.permutation(30)
    assert np.array_equal(oc.gaps(q, k, False, 5, 1), oc.gaps(q, k[:, :, perm], False, 5, 1))


def test_masked_keys_and_unsampled_rows_do_not_matter():
    rng = np.random.default_rng(9)
    q = rng.integers(-128, 128, (1, 1, 12, 8)).astype(np.int8)
    k = rng.integers(-128, 128, (1, 1, 12, 8)).astype(np.int8)
    q[:, :, 11] = 0  # sampled row 11 sees every key but all its scores are 0: gap 0
    base = oc.gaps(q, k, True, 3, 4)  # rows 3, 7, 11
    q2 = q.copy()
    q2[:, :, [0, 1, 2, 4, 5, 6, 8, 9, 10]] = 127  # rows not sampled
    assert np.array_equal(oc.gaps(q2, k, True, 3, 4), base)
    k2 = k.copy()
    k2[:, :, 8:] = 127  # keys 8..11: masked for rows 3 and 7
    assert np.array_equal(oc.gaps(q, k2, True, 3, 4), base)
    k3 = k.copy()
    k3[:, :, 5] = 127  # key 5: visible to row 7, so the gap may change
    assert base[0, 0] > 0


def test_threshold_keeps_the_kth_key_below_index_31(oracle_mod):
    """With c from the rule, every sampled row's K-th largest score gets an
    index <= 30 under the definition's own parameter derivation."""
    rng = np.random.default_rng(10)
    B, H, L, d = 1, 3, 64, 64
    q = rng.integers(-60, 60, (B, H, L, d)).astype(np.int8)
    k = rng.integers(-60, 60, (B, H, L, d)).astype(np.int8)
    s_q = np.array([0.02, 0.03, 0.05], np.float32)
    s_k = np.array([0.04, 0.02, 0.01], np.float32)
    keep, stride = 8, 4
    c, Gh = oc.thresholds(q, k, True, s_q, s_k, False, keep, stride, 0.01, 1e6)
    for h in range(H):
        M, s, D = oracle_mod.index_params(float(s_q[h]), float(s_k[h]), d, float(c[h]))
        assert oracle_mod.index(int(Gh[h]), M, s, D) <= 30
