"""The forward from fp16 / bf16 activations (intattn_forward_fp): quantise q,
k and v on the device, derive the head parameters on the device, run the
integer forward.  Its output must equal, byte for byte, the CPU oracle's
quantisation followed by the oracle forward with the resulting scales, and
the two-step GPU path (intattn_quantize, then intattn_forward with the scales
read back)."""
import numpy as np
import pytest

from oracle import quantize as oq

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


def _inputs(shape_q, shape_kv, dtype, seed):
    import torch
    rng = np.random.default_rng(seed)
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16}[dtype]

    def one(shape, scale):
        x = rng.standard_normal(shape).astype(np.float32) * scale
        ch = rng.choice(shape[-1], size=max(1, shape[-1] // 50), replace=False)
        x[..., ch] *= 8.0  # outlier channels
        return torch.from_numpy(x).to(tdt)

    return one(shape_q, 1.0), one(shape_kv, 1.5), one(shape_kv, 0.7)


CASES = [  # B, H, Lq, Lk, d, causal, per_head, dtype
    (2, 4, 200, 200, 64, False, True, "bf16"),
    (1, 3, 130, 300, 128, False, False, "fp16"),
    (2, 2, 513, 513, 64, True, True, "bf16"),
    (1, 4, 1000, 1000, 128, True, True, "fp16"),
    (3, 2, 64, 256, 64, True, False, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}{}".format(
    *c[:5], "c" if c[5] else "", "h" if c[6] else "", c[7]))
def test_forward_fp_matches_oracle(ia, oracle_mod, case):
    import torch
    B, H, Lq, Lk, d, causal, per_head, dtype = case
    q, k, v = _inputs((B, H, Lq, d), (B, H, Lk, d), dtype, seed=3000 + Lq + Lk + d)
    n = H if per_head else 1
    s_o = np.linspace(0.02, 0.05, n).astype(np.float32)
    clip_c = 8.0 if d == 64 else 10.0
    # oracle: quantise each tensor, then the integer forward with those scales
    cq, sq = oq.quantize(q.float().numpy(), per_head)
    ck, sk = oq.quantize(k.float().numpy(), per_head)
    cv, sv = oq.quantize(v.float().numpy(), per_head)
    want = oracle_mod.forward(cq, ck, cv, per_head, sq, sk, sv, s_o, causal, clip_c)
    scales = torch.zeros(3 * n, dtype=torch.float32, device="cuda")
    out = torch.full((B, H, Lq, d), 0x5A, dtype=torch.int8, device="cuda")
    ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), per_head, s_o, causal, clip_c, out=out, scales_out=scales)
    assert ia.device_error() == ia.OK
    got = out.cpu().numpy()
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} bytes differ from the oracle"
    assert np.array_equal(scales.cpu().numpy(), np.concatenate([sq, sk, sv]))
    # the two-step GPU path gives the same bytes
    c2 = [ia.quantize(t.cuda(), per_head) for t in (q, k, v)]
    sc = ia.Scales(*(s.cpu().numpy() for _, s in c2), s_o, per_head=per_head)
    two = ia.forward(c2[0][0], c2[1][0], c2[2][0], sc, causal, clip_c)
    assert np.array_equal(two.cpu().numpy(), got)


def test_forward_fp_per_head_clip(ia, oracle_mod):
    import torch
    B, H, L, d = 1, 4, 300, 64
    q, k, v = _inputs((B, H, L, d), (B, H, L, d), "bf16", seed=3100)
    s_o = np.full(H, 0.03, np.float32)
    clips = np.array([4.0, 6.0, 8.0, 12.0], np.float32)
    cq, sq = oq.quantize(q.float().numpy(), True)
    ck, sk = oq.quantize(k.float().numpy(), True)
    cv, sv = oq.quantize(v.float().numpy(), True)
    want = np.concatenate([oracle_mod.forward(cq[:, h:h + 1], ck[:, h:h + 1], cv[:, h:h + 1], True, sq[h:h + 1],
                                              sk[h:h + 1], sv[h:h + 1], s_o[h:h + 1], True, float(clips[h]))
                           for h in range(H)], axis=1)
    out = ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), True, s_o, True, 8.0, clip=clips)
    assert ia.device_error() == ia.OK
    assert np.array_equal(out.cpu().numpy(), want)


def test_forward_fp_parameter_out_of_range_is_reported_on_the_device(ia):
    """An output scale so small that the requantisation shift exceeds 62
    is only detectable once the scales exist (on the device): the forward
    writes nothing and intattn_device_error reports PARAM_RANGE; the next
    call is unaffected."""
    import torch
    B, H, L, d = 1, 2, 150, 64
    q, k, v = _inputs((B, H, L, d), (B, H, L, d), "bf16", seed=3200)
    out = torch.full((B, H, L, d), 0x5A, dtype=torch.int8, device="cuda")
    ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), False, [1e-30], False, 8.0, out=out)
    assert ia.device_error() == ia.ERR_PARAM_RANGE
    assert bool((out == 0x5A).all())
    ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), False, [0.03], False, 8.0, out=out)
    assert ia.device_error() == ia.OK
    assert not bool((out == 0x5A).all())


ZP_CASES = [  # B, H, Lq, Lk, d, causal, per_head, dtype, K shift, V shift
    (2, 4, 200, 200, 64, False, True, "bf16", 2.0, -3.0),
    (1, 3, 130, 300, 128, True, False, "fp16", -1.0, 1.5),
    (1, 2, 700, 700, 128, True, True, "bf16", 0.5, 4.0),
]


@pytest.mark.parametrize("case", ZP_CASES, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}{}".format(
    *c[:5], "c" if c[5] else "", "h" if c[6] else "", c[7]))
def test_forward_fp_with_zero_points_matches_oracle(ia, oracle_mod, case):
    """intattn_forward_fp_zp: K and V lopsided (shifted) so that their
    zero-points are far from the middle; equal to oracle quantise (q
    symmetric, k and v asymmetric) + the oracle forward with those
    zero-points, and the zero-points copied out equal the oracle's."""
    import torch
    B, H, Lq, Lk, d, causal, per_head, dtype, ks, vs = case
    q, k, v = _inputs((B, H, Lq, d), (B, H, Lk, d), dtype, seed=3300 + Lq + Lk)
    k = (k.float() + ks).to(k.dtype)
    v = (v.float() + vs).to(v.dtype)
    n = H if per_head else 1
    s_o = np.linspace(0.03, 0.06, n).astype(np.float32)
    cq, sq = oq.quantize(q.float().numpy(), per_head)
    ck, sk, zk = oq.quantize_asym(k.float().numpy(), per_head)
    cv, sv, zv = oq.quantize_asym(v.float().numpy(), per_head)
    want = oracle_mod.forward(cq, ck, cv, per_head, sq, sk, sv, s_o, causal, 8.0, z_k=zk, z_v=zv)
    scales = torch.zeros(3 * n, dtype=torch.float32, device="cuda")
    zps = torch.full((2 * n,), -7, dtype=torch.int32, device="cuda")
    out = ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), per_head, s_o, causal, 8.0, scales_out=scales,
                        zero_points=True, zero_points_out=zps)
    assert ia.device_error() == ia.OK
    assert np.array_equal(scales.cpu().numpy(), np.concatenate([sq, sk, sv]))
    assert np.array_equal(zps.cpu().numpy(), np.concatenate([zk, zv]))
    got = out.cpu().numpy()
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} bytes differ from the oracle"


@pytest.mark.parametrize("zero_points", [False, True], ids=["symmetric", "zero_points"])
def test_forward_fp_full_llama_shape(ia, oracle_mod, zero_points):
    """The headline shape from bf16 activations (B1 H32 L8192 d128, causal,
    per head, clip 10), as the benchmark's forward_fp line runs it: every
    output byte, the scales and the zero-points against oracle quantise +
    the oracle forward.  With zero-points, K and V are shifted so that their
    ranges are lopsided."""
    import torch
    B, H, L, d = 1, 32, 8192, 128
    q, k, v = _inputs((B, H, L, d), (B, H, L, d), "bf16", seed=3700 + int(zero_points))
    if zero_points:
        k = (k.float() + torch.linspace(-3.0, 3.0, H).view(1, H, 1, 1)).to(k.dtype)
        v = (v.float() + torch.linspace(2.0, -2.0, H).view(1, H, 1, 1)).to(v.dtype)
    s_o = np.linspace(0.02, 0.05, H).astype(np.float32)
    cq, sq = oq.quantize(q.float().numpy(), True)
    if zero_points:
        ck, sk, zk = oq.quantize_asym(k.float().numpy(), True)
        cv, sv, zv = oq.quantize_asym(v.float().numpy(), True)
        want = oracle_mod.forward(cq, ck, cv, True, sq, sk, sv, s_o, True, 10.0, z_k=zk, z_v=zv)
    else:
        ck, sk = oq.quantize(k.float().numpy(), True)
        cv, sv = oq.quantize(v.float().numpy(), True)
        want = oracle_mod.forward(cq, ck, cv, True, sq, sk, sv, s_o, True, 10.0)
    scales = torch.zeros(3 * H, dtype=torch.float32, device="cuda")
    zps = torch.full((2 * H,), -7, dtype=torch.int32, device="cuda")
    out = ia.forward_fp(q.cuda(), k.cuda(), v.cuda(), True, s_o, True, 10.0, scales_out=scales,
                        zero_points=zero_points, zero_points_out=zps if zero_points else None)
    assert ia.device_error() == ia.OK
    assert np.array_equal(scales.cpu().numpy(), np.concatenate([sq, sk, sv]))
    if zero_points:
        assert np.array_equal(zps.cpu().numpy(), np.concatenate([zk, zv]))
    got = out.cpu().numpy()
    assert np.array_equal(got, want), f"{int((got != want).sum())} of {got.size} bytes differ from the oracle"
