"""GPU parity of the attention with K / V zero-points (u8 codes; the forum
page's per-layer scale and zero-point, section 动态量化策略) against the CPU
oracle, byte for byte: both prefill kernels, the int8 decode and the
host-buffer forward.  The oracle computes S = q.(k - z_k) and
acc = P.(v - z_v) literally; the kernels run on the codes and subtract
z_v sum P through a correction tile (prefill) or after the reduction
(decode)."""
import numpy as np
import pytest

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


def _inputs(seed, B, H, Lq, Lk, d, per_head, zk, zv):
    """Q int8 N(0, 30); K / V codes: u8 spread around their zero-point (one-
    sided when z is near 0 or 255) when it is given, else int8."""
    rng = np.random.default_rng(seed)
    q = np.clip(np.rint(rng.standard_normal((B, H, Lq, d)) * 30), -128, 127).astype(np.int8)

    def codes(z):
        x = rng.standard_normal((B, H, Lk, d)) * 40
        if z is None:
            return np.clip(np.rint(x), -128, 127).astype(np.int8)
        zz = np.asarray(z).reshape((1, -1, 1, 1)) if per_head else np.asarray(z).reshape(1, 1, 1, 1)
        return np.clip(np.rint(x) + zz, 0, 255).astype(np.uint8)

    k, v = codes(zk), codes(zv)
    n = H if per_head else 1
    s_q = np.full(n, 0.02, np.float32)
    s_k = np.linspace(0.01, 0.03, n).astype(np.float32)
    s_v = np.full(n, 0.05, np.float32)
    s_o = np.linspace(0.02, 0.04, n).astype(np.float32)
    return q, k, v, s_q, s_k, s_v, s_o


def _zp(kind, H, per_head):
    """Zero-points of the test cases: None (int8 codes), or per head / per tensor."""
    if kind is None:
        return None
    vals = {"mid": [128, 100, 150, 90], "edges": [0, 255, 1, 254], "zero": [0, 0, 0, 0]}[kind]
    return np.array([vals[h % 4] for h in range(H)] if per_head else vals[:1], np.int32)


CASES = [  # B, H, Lq, Lk, d, causal, per_head, z_k kind, z_v kind
    (2, 3, 200, 200, 64, False, True, "mid", "mid"),
    (1, 4, 197, 197, 64, False, True, None, "edges"),
    (2, 2, 128, 128, 128, True, False, "edges", None),
    (1, 3, 300, 700, 128, True, True, "mid", "edges"),
    (1, 2, 129, 1500, 64, False, False, "edges", "mid"),
    (2, 4, 256, 256, 128, True, True, "zero", "zero"),
    (1, 2, 1, 1, 64, False, True, "mid", "mid"),
    (1, 4, 333, 512, 64, True, True, None, "mid"),
]


def _variants(ia, Lk):
    vs = [ia.VARIANT_AUTO, ia.VARIANT_THREE_PASS]
    if Lk <= ia.SHORT_ROWS_MAX_KEYS:
        vs.append(ia.VARIANT_SHORT_ROWS)
    return vs


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}-k{}-v{}".format(
    *c[:5], "c" if c[5] else "", "h" if c[6] else "", c[7], c[8]))
def test_prefill_with_zero_points_matches_oracle(ia, oracle_mod, case):
    B, H, Lq, Lk, d, causal, per_head, kk, kv = case
    zk, zv = _zp(kk, H, per_head), _zp(kv, H, per_head)
    q, k, v, s_q, s_k, s_v, s_o = _inputs(sum(case[:5]), B, H, Lq, Lk, d, per_head, zk, zv)
    want = oracle_mod.forward(q, k, v, per_head, s_q, s_k, s_v, s_o, causal, 8.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=per_head, z_k=zk, z_v=zv)
    for variant in _variants(ia, Lk):
        got = ia.forward(_dev(q), _dev(k), _dev(v), sc, causal, 8.0, variant=variant).cpu().numpy()
        assert ia.device_error() == ia.OK
        if not np.array_equal(got, want):
            bad = np.argwhere(got != want)
            raise AssertionError(f"variant {variant}: {len(bad)} bytes differ, first {bad[:3].tolist()}")


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_extreme_codes_with_zero_points(ia, oracle_mod, d):
    """The widest gaps the u8 K range allows (rows of q all -128 or all 127
    against K rows of codes 0 and 255: |gap| up to 128 * 255 * d) and V at
    both ends of its range, with zero-points at the ends."""
    B, H, L = 1, 2, 160
    q = np.where((np.arange(L) % 2 == 0)[:, None], -128, 127).astype(np.int8)[None, None].repeat(H, 1)
    q = np.ascontiguousarray(np.broadcast_to(q, (B, H, L, d)))
    k = np.zeros((B, H, L, d), np.uint8)
    k[:, :, ::3] = 255
    v = np.zeros((B, H, L, d), np.uint8)
    v[:, :, 1::2] = 255
    zk = np.array([0, 255], np.int32)
    zv = np.array([255, 0], np.int32)
    s_q = np.full(H, 0.001, np.float32)
    s_k = np.full(H, 0.001, np.float32)
    s_v = np.full(H, 0.01, np.float32)
    s_o = np.full(H, 0.02, np.float32)
    want = oracle_mod.forward(q, k, v, True, s_q, s_k, s_v, s_o, False, 10.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=True, z_k=zk, z_v=zv)
    for variant in _variants(ia, L):
        got = ia.forward(_dev(q), _dev(k), _dev(v), sc, False, 10.0, variant=variant).cpu().numpy()
        assert np.array_equal(got, want), variant


def test_reexpressed_codes_give_the_symmetric_bytes(ia):
    """int8 K / V shifted to u8 with zero-point 128 run through the kernels
    give the bytes of the symmetric call."""
    B, H, L, d = 2, 3, 400, 128
    q, k, v, s_q, s_k, s_v, s_o = _inputs(5, B, H, L, L, d, True, None, None)
    sym = ia.forward(_dev(q), _dev(k), _dev(v), ia.Scales(s_q, s_k, s_v, s_o, per_head=True), True, 8.0)
    ku = (k.astype(np.int16) + 128).astype(np.uint8)
    vu = (v.astype(np.int16) + 128).astype(np.uint8)
    z = np.full(H, 128, np.int32)
    asym = ia.forward(_dev(q), _dev(ku), _dev(vu), ia.Scales(s_q, s_k, s_v, s_o, per_head=True, z_k=z, z_v=z),
                      True, 8.0)
    assert np.array_equal(sym.cpu().numpy(), asym.cpu().numpy())


DECODE_CASES = [(4, 3, 1000, 1100, 128, True, "mid", "edges"), (2, 2, 4096, 4096, 64, False, "edges", "mid"),
                (3, 4, 37, 64, 128, True, None, "mid"), (1, 2, 513, 600, 64, True, "mid", None)]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "B{}H{}Lk{}Lmax{}d{}-k{}-v{}".format(*c[:5], c[6], c[7]))
def test_decode_with_zero_points_matches_oracle(ia, oracle_mod, case):
    B, H, Lk, Lmax, d, per_head, kk, kv = case
    zk, zv = _zp(kk, H, per_head), _zp(kv, H, per_head)
    q, kc, vc, s_q, s_k, s_v, s_o = _inputs(Lk + d, B, H, 1, Lmax, d, per_head, zk, zv)
    want = oracle_mod.decode(q, kc, vc, per_head, s_q, s_k, s_v, s_o, Lk, 8.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=per_head, z_k=zk, z_v=zv)
    import torch
    ws = torch.full((ia.decode_workspace_size(B, H, Lk, d),), 0x5A, dtype=torch.uint8, device="cuda")
    for _ in range(2):  # the second call reuses the workspace left by the first
        got = ia.decode(_dev(q), _dev(kc), _dev(vc), sc, Lk, 8.0, workspace=ws).cpu().numpy()
        assert ia.device_error() == ia.OK
        assert np.array_equal(got, want)


def test_forward_host_with_zero_points(ia, oracle_mod):
    import torch
    B, H, L, d = 2, 2, 300, 64
    zk, zv = _zp("mid", H, True), _zp("edges", H, True)
    q, k, v, s_q, s_k, s_v, s_o = _inputs(9, B, H, L, L, d, True, zk, zv)
    want = oracle_mod.forward(q, k, v, True, s_q, s_k, s_v, s_o, True, 8.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=True, z_k=zk, z_v=zv)
    pin = lambda a: torch.from_numpy(a).pin_memory()
    out = ia.forward_host(pin(q), pin(k), pin(v), sc, True, 8.0)
    torch.cuda.synchronize()
    assert np.array_equal(out.numpy(), want)


def _pack_u4(c):
    """Unsigned 4-bit codes [..., d] -> bytes [..., d/2], channel 2t in the
    low nibble of byte t (the int4 cache layout)."""
    c = np.asarray(c, dtype=np.uint8)
    assert c.max(initial=0) <= 15
    return (c[..., 0::2] | (c[..., 1::2] << np.uint8(4))).astype(np.uint8)


INT4_CASES = [(4, 3, 1000, 1100, 128, True, "kv"), (2, 2, 4096, 4096, 64, False, "k"),
              (3, 4, 300, 512, 128, True, "v"), (1, 2, 5000, 5000, 128, True, "kv")]


@pytest.mark.parametrize("case", INT4_CASES, ids=lambda c: "B{}H{}Lk{}Lmax{}d{}-{}".format(*c[:5], c[6]))
def test_decode_int4_with_zero_points_matches_oracle(ia, oracle_mod, case):
    """Unsigned int4 codes c in [0, 15] with zero-points 0 .. 15 (lopsided
    code distributions), K, V or both; the other tensor two's complement."""
    from integer_only_quantized_b200 import workloads as wl
    B, H, Lk, Lmax, d, per_head, which = case
    rng = np.random.default_rng(Lk + d + len(which))
    q = np.clip(np.rint(rng.standard_normal((B, H, 1, d)) * 30), -128, 127).astype(np.int8)
    n = H if per_head else 1
    zs = np.array([[0, 15, 7, 3][i % 4] for i in range(n)], np.int32)

    def cache(asym):
        if asym:
            zz = zs.reshape(1, -1, 1, 1) if per_head else zs.reshape(1, 1, 1, 1)
            c = np.clip(np.rint(rng.standard_normal((B, H, Lmax, d)) * 3) + zz, 0, 15).astype(np.uint8)
            return c, _pack_u4(c), zs
        x = rng.integers(-8, 8, (B, H, Lmax, d)).astype(np.int8)
        return x, wl.pack_int4(x), None

    kc, kp, zk = cache("k" in which)
    vc, vp, zv = cache("v" in which)
    s_q = np.full(n, 0.02, np.float32)
    s_k = np.full(n, 0.3, np.float32)
    s_v = np.full(n, 0.4, np.float32)
    s_o = np.full(n, 0.02, np.float32)
    want = oracle_mod.decode(q, kc, vc, per_head, s_q, s_k, s_v, s_o, Lk, 8.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=per_head, z_k=zk, z_v=zv)
    got = ia.decode_int4(_dev(q), _dev(kp), _dev(vp), sc, Lk, 8.0).cpu().numpy()
    assert ia.device_error() == ia.OK
    assert np.array_equal(got, want)


def test_per_head_clips_with_zero_points(ia, oracle_mod):
    """Per-head clip thresholds and per-head zero-points together: each head
    equals the oracle run on that head alone with its threshold."""
    B, H, L, d = 2, 4, 300, 64
    zk, zv = _zp("mid", H, True), _zp("edges", H, True)
    q, k, v, s_q, s_k, s_v, s_o = _inputs(21, B, H, L, L, d, True, zk, zv)
    clips = np.array([4.0, 6.0, 9.0, 12.0], np.float32)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=True, clip=clips, z_k=zk, z_v=zv)
    for variant in (ia.VARIANT_AUTO, ia.VARIANT_THREE_PASS):
        got = ia.forward(_dev(q), _dev(k), _dev(v), sc, True, 8.0, variant=variant).cpu().numpy()
        for h in range(H):
            want = oracle_mod.forward(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], True, s_q[h:h + 1],
                                      s_k[h:h + 1], s_v[h:h + 1], s_o[h:h + 1], True, float(clips[h]),
                                      z_k=zk[h:h + 1], z_v=zv[h:h + 1])
            assert np.array_equal(got[:, h:h + 1], want), (variant, h)


def test_static_scratch_decode_with_zero_points(ia, oracle_mod):
    """The allocation-free decode takes the same zero-point scales."""
    import ctypes

    import torch
    B, H, Lk, Lmax, d = 3, 2, 900, 1024, 128
    zk, zv = _zp("mid", H, True), _zp("edges", H, True)
    q, kc, vc, s_q, s_k, s_v, s_o = _inputs(22, B, H, 1, Lmax, d, True, zk, zv)
    want = oracle_mod.decode(q, kc, vc, True, s_q, s_k, s_v, s_o, Lk, 8.0, z_k=zk, z_v=zv)
    s, keep = ia.Scales(s_q, s_k, s_v, s_o, per_head=True, z_k=zk, z_v=zv)._c()
    qd, kd, vd = _dev(q), _dev(kc), _dev(vc)
    out = torch.full_like(qd, 99)
    rc = ia.lib().intattn_decode_static_scratch(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), ctypes.byref(s), B, H,
                                                Lk, Lmax, d, 8.0, out.data_ptr(),
                                                torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert rc == ia.OK
    assert np.array_equal(out.cpu().numpy(), want)


def test_full_llama_shape_with_per_head_zero_points(ia, oracle_mod):
    """The headline shape (B1 H32 L8192 d128, causal, per head, clip 10) with K
    and V as u8 codes around per-head zero-points that include 0 and 255:
    every output byte against the oracle, which computes q.(k - z_k) and
    P.(v - z_v) literally."""
    B, H, L, d = 1, 32, 8192, 128
    base = [0, 255, 1, 254, 128, 127]
    zk = np.array([base[h] if h < len(base) else (37 * h + 11) % 256 for h in range(H)], np.int32)
    zv = np.array([base[-1 - h] if h < len(base) else (91 * h + 200) % 256 for h in range(H)], np.int32)
    q, k, v, s_q, s_k, s_v, s_o = _inputs(777, B, H, L, L, d, True, zk, zv)
    # a query scale ten times the small cases': over 8192 keys the rows are then
    # peaked enough that the outputs spread over the int8 range (mean |out| ~ 18,
    # a few saturate) instead of averaging to near 0
    s_q = s_q * 10
    want = oracle_mod.forward(q, k, v, True, s_q, s_k, s_v, s_o, True, 10.0, z_k=zk, z_v=zv)
    sc = ia.Scales(s_q, s_k, s_v, s_o, per_head=True, z_k=zk, z_v=zv)
    got = ia.forward(_dev(q), _dev(k), _dev(v), sc, True, 10.0).cpu().numpy()
    assert ia.device_error() == ia.OK
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{len(bad)} of {got.size} bytes differ; first (b, h, i, t) {bad[0].tolist()}")
