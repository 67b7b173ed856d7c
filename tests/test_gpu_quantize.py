"""GPU parity of the quantisation prologue against the numpy oracle: int8
codes and fp32 scales identical, bit for bit; and the whole pipeline
(bf16 -> quantise -> integer attention) against oracle quantise + oracle
attention."""
import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl
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


def _inputs(shape, seed, dtype, spread=(0.01, 30.0), outlier=40.0):
    import torch
    rng = np.random.default_rng(seed)
    B, H, L, d = shape
    x = rng.standard_normal(shape).astype(np.float32) * np.geomspace(*spread, H).astype(np.float32)[None, :, None, None]
    if x.size:
        x.reshape(-1)[rng.integers(0, x.size, size=max(1, x.size // 1000))] *= outlier  # outliers
    t = torch.from_numpy(x).to(dtype)
    return t, t.float().numpy()  # the device input and its exact float32 values


CASES = [((1, 1, 1, 8), False), ((2, 3, 37, 64), True), ((2, 3, 37, 64), False), ((1, 4, 512, 128), True),
         ((3, 2, 1000, 64), True), ((8, 12, 512, 64), False),
         # one CTA over 256 one-vector heads; a full grid over 32 heads of 256K elements;
         # two heads of 2M elements
         ((4, 64, 1, 8), True), ((1, 32, 2048, 128), True), ((1, 2, 16384, 128), True)]


@pytest.mark.parametrize("dtype_name", ["bfloat16", "float16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}L{}d{}{}".format(*c[0], "h" if c[1] else ""))
def test_quantize_parity(ia, case, dtype_name):
    import torch
    shape, per_head = case
    dtype = getattr(torch, dtype_name)
    t, x32 = _inputs(shape, sum(shape) + per_head, dtype)
    codes, scales = ia.quantize(t.cuda(), per_head)
    want_codes, want_scales = oq.quantize(x32, per_head)
    assert np.array_equal(scales.cpu().numpy(), want_scales)
    got = codes.cpu().numpy()
    if not np.array_equal(got, want_codes):
        bad = np.argwhere(got != want_codes)
        raise AssertionError(f"{len(bad)} codes differ, first {bad[:3].tolist()}")


def test_quantize_ties_round_half_to_even(ia):
    import torch
    # amax 127 -> s = 1: x = k + 0.5 ties land on the even neighbour
    vals = [127.0, -127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 62.5, -63.5]
    x = torch.tensor(vals + [0.0] * 6, dtype=torch.bfloat16).reshape(1, 1, 2, 8)
    codes, scales = ia.quantize(x.cuda(), True)
    assert scales.cpu().tolist() == [1.0]
    assert codes.cpu().numpy().ravel()[:10].tolist() == [127, -127, 0, 2, 2, 0, -2, -2, 62, -64]


def test_quantize_product_rounded_before_rint(ia):
    """amax 4.84375, x 2.421875: the exact x * inv lies just below 63.5 but
    the fp32 product is 63.5, a tie that goes to 64; a fused multiply-add
    would give 63."""
    import torch
    x = torch.tensor([4.84375, 2.421875, -2.421875] + [0.0] * 5, dtype=torch.bfloat16).reshape(1, 1, 1, 8)
    inv = np.float32(127.0) / np.float32(4.84375)
    assert np.float32(2.421875) * inv == np.float32(63.5)
    assert 2.421875 * float(inv) < 63.5
    codes, _ = ia.quantize(x.cuda(), True)
    assert codes.cpu().numpy().ravel()[:3].tolist() == [127, 64, -64]
    want, _ = oq.quantize(x.float().numpy(), True)
    assert want.ravel()[:3].tolist() == [127, 64, -64]


def test_quantize_reuses_buffers(ia):
    """Second call into the same code and scale buffers (whose first bytes
    the call uses as scratch) gives the oracle's result again."""
    import torch
    shape = (2, 8, 300, 64)
    out = torch.full(shape, 77, dtype=torch.int8, device="cuda")
    sc = torch.full((8,), 5.0, dtype=torch.float32, device="cuda")
    for seed in (1, 2):
        t, x32 = _inputs(shape, seed, torch.bfloat16)
        ia.quantize(t.cuda(), True, out=out, scales=sc)
        want_codes, want_scales = oq.quantize(x32, True)
        assert np.array_equal(sc.cpu().numpy(), want_scales)
        assert np.array_equal(out.cpu().numpy(), want_codes)


def test_quantize_empty_and_zero(ia):
    import torch
    codes, scales = ia.quantize(torch.zeros((2, 3, 0, 64), dtype=torch.float16, device="cuda"), True)
    assert scales.cpu().tolist() == [1.0, 1.0, 1.0] and codes.numel() == 0
    codes, scales = ia.quantize(torch.zeros((1, 2, 4, 64), dtype=torch.bfloat16, device="cuda"), False)
    assert scales.cpu().tolist() == [1.0] and not codes.cpu().numpy().any()


def test_bf16_pipeline_matches_oracle_pipeline(ia, oracle_mod):
    """bf16 q, k, v -> intattn_quantize -> intattn_forward, against the numpy
    quantise oracle followed by the C attention oracle."""
    import torch
    B, H, L, d = 2, 4, 300, 64
    # activation-like magnitudes (the index multiplier must stay in range)
    tq, q32 = _inputs((B, H, L, d), 11, torch.bfloat16, (0.5, 2.0), 8.0)
    tk, k32 = _inputs((B, H, L, d), 12, torch.bfloat16, (0.5, 2.0), 8.0)
    tv, v32 = _inputs((B, H, L, d), 13, torch.bfloat16, (0.5, 2.0), 8.0)
    (cq, sq), (ck, sk), (cv, sv) = (ia.quantize(t.cuda(), True) for t in (tq, tk, tv))
    s_o = np.full(H, 0.02, np.float32)
    sc = ia.Scales(sq.cpu().numpy(), sk.cpu().numpy(), sv.cpu().numpy(), s_o, per_head=True)
    out = ia.forward(cq, ck, cv, sc, True, 8.0).cpu().numpy()
    assert ia.device_error() == ia.OK
    oq_, osq = oq.quantize(q32, True)
    ok_, osk = oq.quantize(k32, True)
    ov_, osv = oq.quantize(v32, True)
    want = oracle_mod.forward(oq_, ok_, ov_, True, osq, osk, osv, s_o, True, 8.0)
    assert np.array_equal(out, want)
