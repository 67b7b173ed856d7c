"""Pins of the CPU oracle to facts that do not come from the oracle itself.

The pages (IntAttention summaries, "Methodology" item 2) fix the shape of
IndexSoftmax: clip, 32-entry exp table indexed by the integer score gap,
int32 sum, reciprocal by integer multiply and right shift.  The constants and
rounding rules are this build's reading; each test below checks the oracle
against something independent: a closed form derived by hand, an
arbitrary-precision evaluation of the real-valued quantity the integer one
approximates, a library routine, an invariant, or brute force.
"""
import decimal
import math
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x) for x in line.split()])
    return rows


def _dec_exp(x: Fraction) -> decimal.Decimal:
    """exp(x) to 50 digits with Python's decimal module (independent of libm)."""
    with decimal.localcontext() as ctx:
        ctx.prec = 50
        return (decimal.Decimal(x.numerator) / decimal.Decimal(x.denominator)).exp()


# ---------------------------------------------------------------- LUT -----

@pytest.mark.parametrize("c", [4.0, 6.0, 8.0, 10.0, 12.5])
def test_lut_endpoints_monotone_and_rounding(oracle_mod, c):
    lut = oracle_mod.lut(c)
    assert lut.shape == (32,)
    assert lut[0] == 32768            # exp(0) at scale 2^15
    assert lut[31] == 0               # clipped gaps contribute nothing
    assert np.all(np.diff(lut) <= 0), "pseudo-exponentials must not increase"
    big = lut[:31] >= 64            # rounding can only tie entries in the far tail
    assert np.all(np.diff(lut[:31])[big[1:]] < 0)
    cf = Fraction(float(np.float32(c)))
    for i in range(31):
        exact = decimal.Decimal(32768) * _dec_exp(-Fraction(i) * cf / 31)
        assert abs(decimal.Decimal(int(lut[i])) - exact) <= decimal.Decimal("0.5"), (i, lut[i], exact)


def test_lut_ratio_is_geometric(oracle_mod):
    # consecutive entries differ by the factor exp(-c/31) up to rounding
    c = 8.0
    lut = oracle_mod.lut(c).astype(np.float64)
    ratio = math.exp(-c / 31)
    for i in range(1, 31):
        assert abs(lut[i] - lut[i - 1] * ratio) <= 0.5 + 0.5 * ratio + 1e-9


# --------------------------------------------------------- index params ---

SCALE_CASES = [(0.28, 0.28, 64, 8.0), (0.05, 0.02, 128, 10.0), (1.0, 1.0, 64, 8.0),
               (0.011, 0.19, 64, 6.0), (3.0e-4, 2.0e-4, 128, 10.0), (0.9, 0.7, 128, 4.0)]


@pytest.mark.parametrize("sq,sk,d,c", SCALE_CASES)
def test_index_multiplier_approximates_real_ratio(oracle_mod, sq, sk, d, c):
    M, s, D = oracle_mod.index_params(sq, sk, d, c)
    # the real step alpha*31/c, alpha = s_q*s_k/sqrt(d), evaluated independently
    r = float(sq) * float(sk) / math.sqrt(d) * 31.0 / c
    assert 1 <= M <= 2 ** 24 and M <= 2 ** s and 1 <= s <= 26
    assert abs(M - r * 2.0 ** s) <= 0.5 + 1e-6 * r * 2.0 ** s
    # D is the smallest gap whose rounded index reaches 31
    assert oracle_mod.index(D, M, s, D) == 31
    assert oracle_mod.index(D - 1, M, s, D) <= 30
    assert D * M + 2 ** (s - 1) < 2 ** 31


@pytest.mark.parametrize("sq,sk,d,c", SCALE_CASES)
def test_index_is_rounded_scaled_gap(oracle_mod, sq, sk, d, c):
    """idx = round(gap * alpha * 31 / c), clipped to 31 (spec index rule)."""
    M, s, D = oracle_mod.index_params(sq, sk, d, c)
    r = Fraction(float(sq)) * Fraction(float(sk)) * 31 / Fraction(float(c))
    r = r / Fraction(math.sqrt(d))
    err_per_gap = abs(Fraction(M, 2 ** s) - r)
    rng = np.random.default_rng(5)
    gaps = list(range(0, min(3 * D, 5000))) + [int(x) for x in rng.integers(0, 2 ** 22, 2000)]
    prev, prev_g = -1, -2
    for g in sorted(set(gaps)):
        idx = oracle_mod.index(g, M, s, D)
        assert 0 <= idx <= 31
        if g >= D:
            assert idx == 31
        else:
            real = g * r
            assert abs(Fraction(idx) - real) <= Fraction(1, 2) + g * err_per_gap, (g, idx, float(real))
        assert idx >= prev                      # monotone in the gap
        if g == prev_g + 1:
            assert idx - prev <= 1              # M <= 2^s: one gap step, at most one index step
        prev, prev_g = idx, g
    assert oracle_mod.index(0, M, s, D) == 0


def test_index_params_reject_out_of_range(oracle_mod):
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.index_params(0.0, 1.0, 64, 8.0)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.index_params(1.0, 1.0, 64, -1.0)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.index_params(float("nan"), 1.0, 64, 8.0)
    # one integer score step worth more than one LUT step: M would exceed 2^s
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.index_params(40.0, 40.0, 64, 8.0)


# ------------------------------------------------------------ requant -----

def test_requant_golden_half(oracle_mod):
    Mo, so = oracle_mod.requant_params(127.5, 1.0)
    assert (Mo, so) == (2 ** 30, 31)
    for acc, want in _read_golden("requant_half.txt"):
        assert oracle_mod.requant(acc, Mo, so) == want, acc


@pytest.mark.parametrize("sv,so_", [(0.03, 0.01), (1.0, 1.0), (0.25, 0.002), (5e-3, 4e-3)])
def test_requant_multiplier_approximates_real(oracle_mod, sv, so_):
    Mo, so = oracle_mod.requant_params(sv, so_)
    real = Fraction(float(sv)) / (255 * Fraction(float(so_)))
    assert 2 ** 30 <= Mo < 2 ** 31
    assert abs(Fraction(Mo, 2 ** so) - real) <= real * Fraction(1, 2 ** 30)
    rng = np.random.default_rng(1)
    for acc in [int(x) for x in rng.integers(-(2 ** 20), 2 ** 20, 500)]:
        y = oracle_mod.requant(acc, Mo, so)
        want = acc * Fraction(Mo, 2 ** so)
        want = max(-127, min(127, math.floor(want + Fraction(1, 2))))
        assert y == want


# ------------------------------------------------------------- scores -----

def test_scores_match_integer_matmul(oracle_mod):
    rng = np.random.default_rng(2)
    for d in (16, 64, 128):
        q = rng.integers(-128, 128, d, dtype=np.int64).astype(np.int8)
        k = rng.integers(-128, 128, (37, d), dtype=np.int64).astype(np.int8)
        q[0] = -128
        k[:, 0] = -128
        S = oracle_mod.scores(q, k)
        ref = k.astype(np.int64) @ q.astype(np.int64)
        assert np.array_equal(S.astype(np.int64), ref)


# ------------------------------------------------------- IndexSoftmax -----

def test_uniform_rows_golden(oracle_mod):
    lut = oracle_mod.lut(8.0)
    M, s, D = oracle_mod.index_params(0.28, 0.28, 64, 8.0)
    for n, R_want, P_want in _read_golden("uniform_rows.txt"):
        S = np.full(n, 1234, dtype=np.int32)
        P, m, Z, R = oracle_mod.index_softmax(S, M, s, D, lut)
        assert m == 1234 and Z == 32768 * n and R == R_want, n
        assert np.all(P == P_want), n


def test_uniform_rows_with_clipped_tail(oracle_mod):
    """Keys whose gap reaches the clip get E = 0 and change nothing."""
    lut = oracle_mod.lut(8.0)
    M, s, D = oracle_mod.index_params(0.28, 0.28, 64, 8.0)
    for n, _, P_want in _read_golden("uniform_rows.txt")[:6]:
        S = np.concatenate([np.full(n, 500, np.int32), 500 - D - np.arange(9, dtype=np.int32)])
        P, _, Z, _ = oracle_mod.index_softmax(S, M, s, D, lut)
        assert Z == 32768 * n
        assert np.all(P[:n] == P_want) and np.all(P[n:] == 0)


def test_single_dominant_key(oracle_mod):
    lut = oracle_mod.lut(6.0)
    M, s, D = oracle_mod.index_params(0.1, 0.3, 64, 6.0)
    S = np.array([100 - D - 7, 100, 100 - D, 100 - 3 * D, -(2 ** 20)], dtype=np.int32)
    P, m, Z, R = oracle_mod.index_softmax(S, M, s, D, lut)
    assert m == 100 and Z == 32768 and R == 255 * 2 ** 17
    assert P.tolist() == [0, 255, 0, 0, 0]


def test_probabilities_track_real_ratio(oracle_mod):
    """P_j is 255*E_j/Z rounded: |P_j - 255 E_j / Z| <= 1/2 + 2^-17."""
    rng = np.random.default_rng(3)
    lut = oracle_mod.lut(8.0)
    M, s, D = oracle_mod.index_params(0.2, 0.25, 64, 8.0)
    for n in (1, 2, 5, 64, 197, 512, 4096):
        S = rng.integers(-3 * D, 3 * D, n).astype(np.int32)
        P, m, Z, R = oracle_mod.index_softmax(S, M, s, D, lut)
        assert m == S.max()
        E = np.array([lut[oracle_mod.index(int(m - x), M, s, D)] for x in S], dtype=np.int64)
        assert Z == E.sum() and Z >= 32768
        real = Fraction(255) / Z
        for pj, ej in zip(P.tolist(), E.tolist()):
            assert abs(pj - ej * real) <= Fraction(1, 2) + Fraction(1, 2 ** 17)
        nnz = int((E > 0).sum())
        assert abs(int(P.astype(np.int64).sum()) - 255) <= math.ceil(nnz / 2) + 1
        assert P.max() <= 255 and P[S.argmax()] == P.max()


def test_probabilities_follow_softmax(oracle_mod):
    """P/255 vs exact softmax of the logits alpha*S (pages: 'softmax-like')."""
    rng = np.random.default_rng(4)
    c = 8.0
    sq, sk, d = 0.05, 0.05, 64
    lut = oracle_mod.lut(c)
    M, s, D = oracle_mod.index_params(sq, sk, d, c)
    alpha = sq * sk / math.sqrt(d)
    for _ in range(20):
        S = rng.integers(-2000, 2000, 16).astype(np.int32)
        P, *_ = oracle_mod.index_softmax(S, M, s, D, lut)
        x = alpha * S.astype(np.float64)
        ex = np.exp(x - x.max())
        ref = ex / ex.sum()
        # half a LUT step is a factor exp(c/62); plus u8 rounding
        assert np.max(np.abs(P / 255.0 - ref)) <= 0.14 * ref.max() + 2.0 / 255


# ------------------------------------------------------ full attention ----

def _fp_attention(q, k, v, sq, sk, sv, causal):
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    qf = q.astype(np.float64) * sq
    kf = k.astype(np.float64) * sk
    vf = v.astype(np.float64) * sv
    logits = np.einsum("bhid,bhjd->bhij", qf, kf) / math.sqrt(d)
    if causal:
        mask = np.arange(Lk)[None, :] > (np.arange(Lq)[:, None] + Lk - Lq)
        logits = np.where(mask, -np.inf, logits)
    logits -= logits.max(-1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(-1, keepdims=True)
    return np.einsum("bhij,bhjd->bhid", p, vf)


def _quant(x):
    s = np.float32(np.abs(x).max() / 127.0)
    return np.clip(np.rint(x / np.float64(s)), -127, 127).astype(np.int8), s


@pytest.mark.parametrize("L,d,causal,c", [(8, 16, False, 8.0), (32, 16, True, 8.0),
                                          (32, 64, False, 8.0), (24, 64, True, 6.0),
                                          (32, 64, False, 10.0)])
def test_brute_force_against_fp_attention(oracle_mod, L, d, causal, c):
    """De-quantised oracle output vs fp64 softmax attention on tiny inputs:
    cosine >= 0.995 and max-abs error <= 0.05 * max|V|."""
    rng = np.random.default_rng(100 + L + d)
    B, H = 2, 3
    xs = []
    for _ in range(3):
        x = rng.standard_normal((B, H, L, d)).astype(np.float32)
        x[:, :, :, rng.choice(d, max(1, d // 50), replace=False)] *= 8.0
        xs.append(x)
    (q, sq), (k, sk), (v, sv) = [_quant(x) for x in xs]
    ref = _fp_attention(q, k, v, float(sq), float(sk), float(sv), causal)
    so = np.float32(np.abs(ref).max() / 127.0)
    out = oracle_mod.forward(q, k, v, False, sq, sk, sv, so, causal, c)
    got = out.astype(np.float64) * float(so)
    cos = float((got * ref).sum() / (np.linalg.norm(got) * np.linalg.norm(ref)))
    vmax = float(np.abs(v).max()) * float(sv)
    assert cos >= 0.995, cos
    assert np.abs(got - ref).max() <= 0.05 * vmax, (np.abs(got - ref).max(), vmax)


def test_single_key_reproduces_v(oracle_mod):
    """Lk = 1: P = 255, and with s_v = s_o the output is V itself."""
    rng = np.random.default_rng(7)
    q = rng.integers(-127, 128, (1, 2, 1, 64)).astype(np.int8)
    k = rng.integers(-127, 128, (1, 2, 1, 64)).astype(np.int8)
    v = rng.integers(-127, 128, (1, 2, 1, 64)).astype(np.int8)
    out = oracle_mod.forward(q, k, v, False, 0.1, 0.1, 0.02, 0.02, False, 8.0)
    assert np.array_equal(out, v)
    out2 = oracle_mod.forward(q, k, v, False, 0.1, 0.1, 0.04, 0.02, False, 8.0)
    assert np.array_equal(out2, np.clip(2 * v.astype(np.int32), -127, 127).astype(np.int8))


def test_causal_rows_ignore_masked_keys(oracle_mod):
    rng = np.random.default_rng(8)
    B, H, Lq, Lk, d = 1, 2, 9, 13, 16
    q = rng.integers(-127, 128, (B, H, Lq, d)).astype(np.int8)
    k = rng.integers(-127, 128, (B, H, Lk, d)).astype(np.int8)
    v = rng.integers(-127, 128, (B, H, Lk, d)).astype(np.int8)
    base = oracle_mod.forward(q, k, v, False, 0.02, 0.02, 0.02, 0.005, True, 8.0)
    off = Lk - Lq
    for i in range(Lq):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, i + off + 1:] = 127
        v2[:, :, i + off + 1:] = -127
        out = oracle_mod.forward(q, k2, v2, False, 0.02, 0.02, 0.02, 0.005, True, 8.0)
        assert np.array_equal(out[:, :, i], base[:, :, i])
    # and a key inside the window does matter for the last row
    k3 = k.copy()
    k3[:, :, 0] = -k3[:, :, 0]
    v3 = v.copy()
    v3[:, :, 0] = 127
    out3 = oracle_mod.forward(q, k3, v3, False, 0.02, 0.02, 0.02, 0.005, True, 8.0)
    assert not np.array_equal(out3[:, :, -1], base[:, :, -1])


def test_row_permutation_equivariance(oracle_mod):
    """Permuting key/value rows together leaves a non-causal output unchanged;
    permuting query rows permutes the output rows."""
    rng = np.random.default_rng(9)
    q = rng.integers(-127, 128, (1, 2, 11, 32)).astype(np.int8)
    k = rng.integers(-127, 128, (1, 2, 17, 32)).astype(np.int8)
    v = rng.integers(-127, 128, (1, 2, 17, 32)).astype(np.int8)
    args = (False, 0.03, 0.02, 0.05, 0.01, False, 8.0)
    base = oracle_mod.forward(q, k, v, *args)
    pk = rng.permutation(17)
    pq = rng.permutation(11)
    out = oracle_mod.forward(q[:, :, pq], k[:, :, pk], v[:, :, pk], *args)
    assert np.array_equal(out, base[:, :, pq])


def test_linearity_in_v_before_requant(oracle_mod):
    """Negating V negates the output exactly when the requant rounding is odd-
    symmetric: check with s_v = s_o*255*2^-k so the product is exact."""
    rng = np.random.default_rng(10)
    q = rng.integers(-127, 128, (1, 1, 5, 16)).astype(np.int8)
    k = rng.integers(-127, 128, (1, 1, 9, 16)).astype(np.int8)
    v = rng.integers(-127, 128, (1, 1, 9, 16)).astype(np.int8)
    # m_o = s_v/(255 s_o) = 2^-8 exactly -> out = floor(acc/256 + 1/2)
    sv, so_ = 255.0 / 256.0, 1.0
    out = oracle_mod.forward(q, k, v, False, 0.02, 0.02, sv, so_, False, 8.0)
    # independent: P from index_softmax, acc with numpy, rounding with Fraction
    lut = oracle_mod.lut(8.0)
    M, s, D = oracle_mod.index_params(0.02, 0.02, 16, 8.0)
    for i in range(5):
        S = (k[0, 0].astype(np.int64) @ q[0, 0, i].astype(np.int64)).astype(np.int32)
        P, *_ = oracle_mod.index_softmax(S, M, s, D, lut)
        acc = P.astype(np.int64) @ v[0, 0].astype(np.int64)
        want = [max(-127, min(127, math.floor(Fraction(int(a), 256) + Fraction(1, 2)))) for a in acc]
        assert out[0, 0, i].tolist() == want


def test_rows_and_decode_agree_with_forward(oracle_mod):
    rng = np.random.default_rng(11)
    B, H, L, d = 2, 3, 21, 32
    q = rng.integers(-127, 128, (B, H, L, d)).astype(np.int8)
    k = rng.integers(-127, 128, (B, H, L, d)).astype(np.int8)
    v = rng.integers(-127, 128, (B, H, L, d)).astype(np.int8)
    sc = dict(per_head=True, s_q=[0.02, 0.03, 0.01], s_k=[0.02, 0.01, 0.04],
              s_v=[0.05, 0.02, 0.03], s_o=[0.01, 0.01, 0.02])
    full = oracle_mod.forward(q, k, v, sc["per_head"], sc["s_q"], sc["s_k"], sc["s_v"],
                              sc["s_o"], True, 8.0)
    rows = np.array([[1, 2, 20], [0, 0, 0], [1, 1, 7]])
    got = oracle_mod.forward_rows(q, k, v, True, sc["s_q"], sc["s_k"], sc["s_v"], sc["s_o"],
                                  True, 8.0, rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(got[r], full[b, h, i])
    # decode of the last query row over a cache with spare capacity = causal last row
    Lmax = L + 5
    kc = np.zeros((B, H, Lmax, d), np.int8)
    vc = np.zeros((B, H, Lmax, d), np.int8)
    kc[:, :, :L] = k
    vc[:, :, :L] = v
    kc[:, :, L:] = 127
    vc[:, :, L:] = 99
    dec = oracle_mod.decode(q[:, :, -1:], kc, vc, True, sc["s_q"], sc["s_k"], sc["s_v"],
                            sc["s_o"], L, 8.0)
    assert np.array_equal(dec[:, :, 0], full[:, :, -1])


def test_per_head_with_equal_scales_matches_per_tensor(oracle_mod):
    rng = np.random.default_rng(12)
    q = rng.integers(-127, 128, (1, 4, 6, 16)).astype(np.int8)
    k = rng.integers(-127, 128, (1, 4, 6, 16)).astype(np.int8)
    v = rng.integers(-127, 128, (1, 4, 6, 16)).astype(np.int8)
    a = oracle_mod.forward(q, k, v, False, 0.03, 0.02, 0.05, 0.01, False, 8.0)
    b = oracle_mod.forward(q, k, v, True, [0.03] * 4, [0.02] * 4, [0.05] * 4, [0.01] * 4,
                           False, 8.0)
    assert np.array_equal(a, b)


def test_forward_rejects_bad_arguments(oracle_mod):
    q = np.zeros((1, 1, 4, 16), np.int8)
    k = np.zeros((1, 1, 3, 16), np.int8)
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(q, k, k, False, 0.1, 0.1, 0.1, 0.1, True, 8.0)  # causal, Lq > Lk
    with pytest.raises(oracle_mod.OracleError):
        oracle_mod.forward(q, k, k, False, 0.1, 0.1, 0.0, 0.1, False, 8.0)  # zero scale
