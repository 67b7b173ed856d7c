"""GPU parity: the sm_100a kernels, called through the C ABI, against the CPU
oracle on the same seeded inputs.  int8 outputs must be identical byte for
byte (the whole path is integer arithmetic)."""
import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ia():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from integer_only_quantized_b200 import build
    build.build()
    import integer_only_quantized_b200 as mod
    mod.lib()
    return mod


def _dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _gpu_forward(ia, x, w, guard=0):
    """Run the C-ABI forward; with guard > 0 the output sits between canary bands."""
    import torch
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    q, k, v = _dev(x.q), _dev(x.k), _dev(x.v)
    n = x.q.size
    buf = torch.full((n + 2 * guard,), 0x5A, dtype=torch.int8, device="cuda")
    out = buf[guard:guard + n].view(x.q.shape)
    ia.forward(q, k, v, sc, w.causal, w.clip_c, out=out)
    assert ia.device_error() == ia.OK
    if guard:
        b = buf.cpu().numpy()
        assert np.all(b[:guard] == 0x5A) and np.all(b[guard + n:] == 0x5A), "write outside out"
    return out.cpu().numpy()


def _oracle_forward(oracle_mod, x, w):
    return oracle_mod.forward(x.q, x.k, x.v, w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.causal, w.clip_c)


def _assert_equal(got, want, what):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(bad)} of {got.size} bytes differ; first at {bad[:5].tolist()} "
                             f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")


# ----------------------------------------------------- benchmark workloads

@pytest.mark.parametrize("name", ["bert_base_l128", "bert_base_b8_l512", "vit_b16_l197"])
def test_workload_full_parity(ia, oracle_mod, name):
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w)
    got = _gpu_forward(ia, x, w, guard=4096)
    _assert_equal(got, _oracle_forward(oracle_mod, x, w), name)


def _sample_rows(w, rng, n_random=256):
    rows = set()
    Lq = w.Lq
    special = sorted({i for i in (0, 1, 126, 127, 128, 129, 255, 256, Lq // 2, Lq - 129, Lq - 128,
                                  Lq - 2, Lq - 1) if 0 <= i < Lq})
    for b in {0, w.B - 1}:
        for h in {0, w.H - 1}:
            for i in special:
                rows.add((b, h, i))
    for _ in range(n_random):
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.H)), int(rng.integers(Lq))))
    return np.array(sorted(rows), dtype=np.int32)


@pytest.mark.parametrize("name", ["gpt2_small_causal_l2048", "llama7b_causal_l8192"])
def test_workload_full_parity_causal(ia, oracle_mod, name):
    """Full-size causal workloads, launched exactly as the benchmark does.
    A sample of special rows (tile edges, first and last rows and heads) is
    checked first, so a mismatch there is reported quickly; then every output
    byte is compared with the oracle run over all rows on every host core."""
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w)
    got = _gpu_forward(ia, x, w, guard=4096)
    rows = _sample_rows(w, np.random.default_rng(w.seed))
    want = oracle_mod.forward_rows(x.q, x.k, x.v, w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.causal,
                                   w.clip_c, rows)
    sampled = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    if not np.array_equal(sampled, want):
        r = int(np.argwhere((sampled != want).any(axis=1))[0][0])
        raise AssertionError(f"{name}: sampled row (b, h, i) = {rows[r].tolist()} differs from the oracle")
    _assert_equal(got, _oracle_forward(oracle_mod, x, w), name)
    # the same call twice gives the same bytes
    again = _gpu_forward(ia, x, w)
    _assert_equal(again, got, name + " (determinism)")


def test_decode_workload_full_parity(ia, oracle_mod):
    w = wl.WORKLOADS["llama7b_decode_b64_lk4096"]
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    out = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, w.Lk, w.clip_c)
    assert ia.device_error() == ia.OK
    want = oracle_mod.decode(x.q, x.k, x.v, w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.Lk, w.clip_c)
    _assert_equal(out.cpu().numpy(), want, w.name)


# ----------------------------------------------------------- shape sweep

SWEEP = [
    # (B, H, Lq, Lk, d, causal, per_head, dist)
    (1, 1, 1, 1, 64, False, False, "normal"),
    (1, 2, 1, 1, 128, True, True, "normal"),
    (2, 3, 31, 31, 64, True, False, "normal"),
    (1, 2, 127, 127, 128, False, True, "student_t4"),
    (1, 2, 128, 128, 64, True, False, "normal"),
    (1, 2, 129, 129, 128, True, True, "normal"),
    (2, 2, 197, 197, 64, False, True, "student_t4"),
    (1, 3, 255, 255, 128, False, False, "normal"),
    (1, 2, 256, 256, 64, True, True, "normal"),
    (1, 2, 511, 511, 64, False, False, "normal"),
    (1, 2, 513, 513, 128, True, False, "normal"),
    (1, 1, 1000, 1000, 128, True, True, "normal"),
    (1, 2, 64, 300, 64, True, False, "normal"),     # Lq < Lk, bottom-right causal
    (1, 2, 130, 700, 128, False, True, "normal"),   # cross attention, ragged
    (1, 2, 1, 777, 64, True, False, "normal"),      # one query row sees every key
    (3, 1, 200, 200, 128, False, False, "student_t4"),
]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "h" if c[6] else ""))
def test_shape_sweep(ia, oracle_mod, case):
    B, H, Lq, Lk, d, causal, per_head, dist = case
    w = wl.custom_workload("sweep", B, H, Lq, Lk, d, causal, per_head=per_head, dist=dist,
                           clip_c=8.0 if d == 64 else 10.0, index=300 + Lq + Lk + d)
    x = wl.make_inputs(w)
    got = _gpu_forward(ia, x, w, guard=1024)
    _assert_equal(got, _oracle_forward(oracle_mod, x, w), str(case))


@pytest.mark.parametrize("d", [64, 128])
def test_extreme_codes(ia, oracle_mod, d):
    """-128 codes everywhere (largest |S| = 128^2 d), and rows of equal scores."""
    import dataclasses
    w = wl.custom_workload("extreme", 1, 2, 200, 200, d, True, index=700 + d)
    x = wl.make_inputs(w)
    x = dataclasses.replace(x, q=np.full_like(x.q, -128), k=np.full_like(x.k, -128))
    _assert_equal(_gpu_forward(ia, x, w), _oracle_forward(oracle_mod, x, w), "all -128")
    rng = np.random.default_rng(d)
    k = np.where(rng.random(x.k.shape) < 0.5, -128, 127).astype(np.int8)
    v = np.where(rng.random(x.v.shape) < 0.5, -128, 127).astype(np.int8)
    x2 = dataclasses.replace(x, q=np.full_like(x.q, 127), k=k, v=v)
    _assert_equal(_gpu_forward(ia, x2, w), _oracle_forward(oracle_mod, x2, w), "+-extremes")
    x3 = dataclasses.replace(x, q=np.zeros_like(x.q))  # every score 0: uniform rows
    _assert_equal(_gpu_forward(ia, x3, w), _oracle_forward(oracle_mod, x3, w), "uniform rows")


@pytest.mark.parametrize("clip_c", [0.5, 3.0, 30.0])
def test_clip_extremes(ia, oracle_mod, clip_c):
    """Tiny clip (most keys clipped to index 31) and huge clip (none)."""
    w = wl.custom_workload("clip", 2, 2, 300, 300, 64, False, clip_c=clip_c, index=800)
    x = wl.make_inputs(w)
    _assert_equal(_gpu_forward(ia, x, w), _oracle_forward(oracle_mod, x, w), f"c={clip_c}")


# ---------------------------------------------------------------- decode

DECODE_SWEEP = [
    (1, 1, 1, 1, 64), (2, 3, 100, 160, 128), (1, 2, 511, 511, 64), (1, 2, 512, 512, 128),
    (2, 2, 513, 600, 64), (3, 2, 1500, 2048, 128), (1, 4, 4096, 4100, 64), (2, 1, 9000, 9000, 128),
]


@pytest.mark.parametrize("case", DECODE_SWEEP, ids=lambda c: "B{}H{}Lk{}Lmax{}d{}".format(*c))
def test_decode_sweep(ia, oracle_mod, case):
    import torch
    B, H, Lk, Lmax, d = case
    w = wl.custom_workload("dec", B, H, 1, Lk, d, False, per_head=True, clip_c=10.0,
                           index=500 + Lk + d, decode=True, Lmax=Lmax)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True)
    # a workspace full of garbage: the kernels must not depend on its contents
    ws = torch.randint(0, 255, (ia.decode_workspace_size(B, H, Lk, d),), dtype=torch.uint8, device="cuda")
    out = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, Lk, w.clip_c, workspace=ws)
    assert ia.device_error() == ia.OK
    want = oracle_mod.decode(x.q, x.k, x.v, True, x.s_q, x.s_k, x.s_v, x.s_o, Lk, w.clip_c)
    _assert_equal(out.cpu().numpy(), want, str(case))
    # second call on the same workspace
    out2 = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, Lk, w.clip_c, workspace=ws)
    _assert_equal(out2.cpu().numpy(), want, str(case) + " (reused workspace)")


def test_decode_matches_prefill_last_row(ia):
    """Decode of query row i over the first Lk cache rows == row i of the
    causal prefill (same definition, independent kernels)."""
    w = wl.custom_workload("dec_vs_prefill", 2, 3, 700, 700, 128, True, per_head=True, clip_c=10.0,
                           index=950)
    x = wl.make_inputs(w)
    pre = _gpu_forward(ia, x, w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True)
    for i in (0, 350, 699):
        out = ia.decode(_dev(x.q[:, :, i:i + 1]), _dev(x.k), _dev(x.v), sc, i + 1, w.clip_c)
        _assert_equal(out.cpu().numpy()[:, :, 0], pre[:, :, i], f"row {i}")


# ---------------------------------------------- kernel variants, short rows

def _variant_forward(ia, x, w, variant, guard=1024):
    import torch
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    q, k, v = _dev(x.q), _dev(x.k), _dev(x.v)
    n = x.q.size
    buf = torch.full((n + 2 * guard,), 0x5A, dtype=torch.int8, device="cuda")
    out = buf[guard:guard + n].view(x.q.shape)
    ia.forward(q, k, v, sc, w.causal, w.clip_c, out=out, variant=variant)
    assert ia.device_error() == ia.OK
    b = buf.cpu().numpy()
    assert np.all(b[:guard] == 0x5A) and np.all(b[guard + n:] == 0x5A), "write outside out"
    return out.cpu().numpy()


SHORT_SWEEP = [
    # (B, H, Lq, Lk, d, causal, per_head, dist): every Lk <= 512
    (1, 1, 1, 1, 64, False, False, "normal"),
    (2, 3, 32, 32, 128, False, True, "normal"),
    (1, 2, 33, 33, 64, True, False, "normal"),
    (2, 2, 127, 127, 64, False, True, "student_t4"),
    (1, 2, 129, 129, 128, True, True, "normal"),
    (3, 4, 197, 197, 64, False, True, "student_t4"),
    (1, 3, 256, 256, 128, False, False, "normal"),
    (1, 3, 257, 257, 64, True, False, "normal"),
    (2, 2, 300, 300, 128, False, True, "normal"),
    (1, 2, 384, 384, 64, True, True, "normal"),
    (1, 2, 511, 511, 128, True, False, "normal"),
    (2, 3, 512, 512, 64, False, False, "normal"),
    (1, 2, 100, 512, 64, True, False, "normal"),     # Lq < Lk, bottom-right causal
    (1, 2, 600, 200, 128, False, True, "normal"),    # cross attention, more queries than keys
    (8, 40, 512, 512, 64, True, True, "normal"),     # 1280 tiles: CTAs mix 1..4 key tiles
    (8, 40, 256, 256, 128, True, True, "normal"),    # 640 tiles: CTAs mix 1 and 2 key tiles
    (4, 30, 250, 250, 64, True, False, "normal"),    # causal, ragged: the second q tile has 122 rows
    (24, 12, 197, 197, 64, False, True, "student_t4"),  # 576 tiles: several rounds of resident tiles
]


@pytest.mark.parametrize("case", SHORT_SWEEP, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "h" if c[6] else ""))
def test_short_row_variants_match_oracle(ia, oracle_mod, case):
    """Rows of at most 512 keys: the short-row kernel (scores resident in
    tensor memory, up to 256 keys), the three-pass kernel and the automatic
    choice must each give the oracle's bytes."""
    B, H, Lq, Lk, d, causal, per_head, dist = case
    w = wl.custom_workload("short", B, H, Lq, Lk, d, causal, per_head=per_head, dist=dist,
                           clip_c=8.0 if d == 64 else 10.0, index=2000 + Lq + 3 * Lk + d + B)
    x = wl.make_inputs(w)
    want = _oracle_forward(oracle_mod, x, w)
    variants = [ia.VARIANT_AUTO, ia.VARIANT_THREE_PASS]
    if Lk <= ia.SHORT_ROWS_MAX_KEYS:
        variants.append(ia.VARIANT_SHORT_ROWS)
    for variant in variants:
        _assert_equal(_variant_forward(ia, x, w, variant), want, f"{case} variant {variant}")


@pytest.mark.parametrize("name", ["bert_base_l128", "bert_base_b8_l512", "vit_b16_l197"])
def test_workload_both_variants(ia, oracle_mod, name):
    """The short-row workloads through each kernel that takes them."""
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w)
    want = _oracle_forward(oracle_mod, x, w)
    variants = [ia.VARIANT_THREE_PASS] + ([ia.VARIANT_SHORT_ROWS] if w.Lk <= ia.SHORT_ROWS_MAX_KEYS else [])
    for variant in variants:
        _assert_equal(_variant_forward(ia, x, w, variant, guard=4096), want, f"{name} variant {variant}")


@pytest.mark.parametrize("d", [64, 128])
def test_short_rows_extreme_codes(ia, oracle_mod, d):
    """Largest |S| and all-equal rows through the short-row kernel."""
    import dataclasses
    w = wl.custom_workload("short_extreme", 2, 3, 250, 250, d, True, index=2700 + d)
    x = wl.make_inputs(w)
    cases = [dataclasses.replace(x, q=np.full_like(x.q, -128), k=np.full_like(x.k, -128)),
             dataclasses.replace(x, q=np.zeros_like(x.q))]
    for xx in cases:
        _assert_equal(_variant_forward(ia, xx, w, ia.VARIANT_SHORT_ROWS), _oracle_forward(oracle_mod, xx, w),
                      "extreme")


# ------------------------------------------------ the largest key count (Lk = 65535)

@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_max_key_length_all_equal_rows(ia, oracle_mod, causal):
    """Lk = 65535, the largest the definition allows.  Head 0 has q = 0, so
    every score is 0 and each row's sum is 32768 times its visible keys, up
    to 32768 * 65535 = 2^31 - 32768 (the bound that limits Lk; every P is
    then 0).  Head 1 keeps random queries at ten times the query scale, so
    its rows are peaked enough for outputs away from 0.  Both the automatic
    kernel and the three-pass kernel against the oracle."""
    import dataclasses
    w = wl.custom_workload("max_lk_equal", 1, 2, 130, 65535, 64, causal, per_head=True, index=4100 + causal)
    x = wl.make_inputs(w)
    q = x.q.copy()
    q[:, 0] = 0
    s_q = x.s_q.copy()
    s_q[1] *= 10
    xx = dataclasses.replace(x, q=q, s_q=s_q)
    want = _oracle_forward(oracle_mod, xx, w)
    for variant in (ia.VARIANT_AUTO, ia.VARIANT_THREE_PASS):
        _assert_equal(_variant_forward(ia, xx, w, variant), want, f"Lk 65535 all-equal, variant {variant}")


def test_max_key_length_causal_prefill(ia, oracle_mod):
    """Lq = Lk = 65535, causal, random codes: 512 query tiles of 1..512 key
    tiles, the last one ragged (127 rows), every output byte."""
    w = wl.custom_workload("max_lk_causal", 1, 1, 65535, 65535, 64, True, index=4110)
    x = wl.make_inputs(w)
    _assert_equal(_gpu_forward(ia, x, w, guard=4096), _oracle_forward(oracle_mod, x, w), "Lq = Lk = 65535 causal")


@pytest.mark.parametrize("bits", [8, 4])
def test_max_key_length_decode(ia, oracle_mod, bits):
    """One query over 65535 cached keys (128 split-K chunks for int8), int8 and int4 caches."""
    w = wl.custom_workload("max_lk_decode", 2, 2, 1, 65535, 128, False, per_head=True, clip_c=10.0,
                           index=4120 + bits, decode=True, Lmax=65536, kv_bits=bits)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True)
    if bits == 8:
        out = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, w.Lk, w.clip_c)
    else:
        out = ia.decode_int4(_dev(x.q), _dev(wl.pack_int4(x.k)), _dev(wl.pack_int4(x.v)), sc, w.Lk, w.clip_c)
    assert ia.device_error() == ia.OK
    want = oracle_mod.decode(x.q, x.k, x.v, True, x.s_q, x.s_k, x.s_v, x.s_o, w.Lk, w.clip_c)
    _assert_equal(out.cpu().numpy(), want, f"decode Lk 65535 int{bits}")
