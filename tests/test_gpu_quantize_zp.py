"""GPU parity of the asymmetric quantisation prologue (intattn_quantize_zp)
against the numpy oracle (oracle.quantize.quantize_asym): u8 codes, fp32
scales and int32 zero-points identical, bit for bit."""
import os

import numpy as np
import pytest

from oracle import quantize as oq

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_zero_point.txt")


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


def _inputs(shape, seed, dtype, shift=0.0):
    """Heads of different spread, each shifted (so ranges are one-sided or
    lopsided), with rare outliers; returns the device tensor and its exact
    float32 values."""
    import torch
    rng = np.random.default_rng(seed)
    B, H, L, d = shape
    x = rng.standard_normal(shape).astype(np.float32) * np.geomspace(0.01, 30.0, H).astype(np.float32)[None, :, None, None]
    x += (np.linspace(-1.0, 1.0, H).astype(np.float32) * shift * np.geomspace(0.01, 30.0, H).astype(np.float32))[None, :, None, None]
    if x.size:
        x.reshape(-1)[rng.integers(0, x.size, size=max(1, x.size // 1000))] *= 8.0
    t = torch.from_numpy(x).to(dtype)
    return t, t.float().numpy()


CASES = [((1, 1, 1, 8), False, 0.0), ((2, 3, 37, 64), True, 2.0), ((2, 3, 37, 64), False, 0.5),
         ((1, 4, 512, 128), True, 3.0), ((3, 2, 1000, 64), True, 0.0), ((8, 12, 512, 64), False, 1.0),
         ((4, 64, 1, 8), True, 2.5), ((1, 32, 2048, 128), True, 1.5), ((1, 2, 16384, 128), True, 4.0)]


def _check(ia, t, x32, per_head):
    codes, scales, zps = ia.quantize_zp(t.cuda(), per_head)
    wc, ws, wz = oq.quantize_asym(x32, per_head)
    assert np.array_equal(scales.cpu().numpy(), ws), (scales.cpu().numpy()[:4], ws[:4])
    assert np.array_equal(zps.cpu().numpy(), wz), (zps.cpu().numpy()[:4], wz[:4])
    got = codes.cpu().numpy()
    if not np.array_equal(got, wc):
        bad = np.argwhere(got != wc)
        raise AssertionError(f"{len(bad)} codes differ, first {bad[:3].tolist()}: got {got[tuple(bad[0])]} "
                             f"want {wc[tuple(bad[0])]}")


@pytest.mark.parametrize("dtype_name", ["bfloat16", "float16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}L{}d{}{}s{}".format(*c[0], "h" if c[1] else "", c[2]))
def test_quantize_zp_parity(ia, case, dtype_name):
    import torch
    shape, per_head, shift = case
    t, x32 = _inputs(shape, sum(shape) + per_head + int(10 * shift), getattr(torch, dtype_name), shift)
    _check(ia, t, x32, per_head)


def test_quantize_zp_golden_cases(ia):
    """The hand-derived cases: ties to even, the clamp at 255, a positive-only
    head, the reciprocal-product tie and an odd zero-point (fp16, padded to
    whole 16-byte vectors with zeros, which change no range)."""
    import torch
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        key, v = line.split(":")
        vals[key.strip()] = [float(x) for x in v.split()]
    for case in ("ties", "clamp", "positive", "recip", "odd"):
        x = np.zeros(16, np.float32)
        n = len(vals[case + "_values"])
        x[:n] = vals[case + "_values"]
        t = torch.from_numpy(x.reshape(1, 1, 2, 8)).to(torch.float16)
        codes, s, z = ia.quantize_zp(t.cuda(), False)
        got = codes.cpu().numpy().ravel()[:n].tolist()
        assert got == [int(c) for c in vals[case + "_codes"]], case
        assert float(s.cpu()[0]) == vals[case + "_scale"][0], case
        assert int(z.cpu()[0]) == int(vals[case + "_zero_point"][0]), case


def test_quantize_zp_one_sided_and_zero(ia):
    import torch
    x = np.abs(np.random.default_rng(3).standard_normal((1, 3, 64, 64))).astype(np.float32) + 0.5
    x[:, 1] *= -1.0
    x[:, 2] = 0.0
    t = torch.from_numpy(x).to(torch.bfloat16)
    _check(ia, t, t.float().numpy(), True)
    codes, s, z = ia.quantize_zp(t.cuda(), True)
    assert z.cpu().numpy().tolist() == [0, 255, 0]
    assert s.cpu().numpy()[2] == 1.0 and not codes[:, 2].any()


def test_quantize_zp_empty(ia):
    import torch
    t = torch.zeros((0, 4, 16, 64), dtype=torch.float16, device="cuda")
    s = torch.full((4,), 7.0, device="cuda")
    z = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    codes, s, z = ia.quantize_zp(t, True, scales=s, zero_points=z)
    assert s.cpu().numpy().tolist() == [1.0] * 4 and z.cpu().numpy().tolist() == [0] * 4


def test_quantize_zp_reuses_buffers_and_leaves_symmetric_alone(ia):
    """Back-to-back calls on the same buffers (stale maxima and counters are
    cleared per call); the symmetric entry point is unchanged by the option."""
    import torch
    t1, x1 = _inputs((2, 4, 300, 64), 41, torch.float16, 2.0)
    t2, x2 = _inputs((2, 4, 300, 64), 42, torch.float16, -1.0)
    out = torch.empty(t1.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, device="cuda")
    z = torch.empty(4, dtype=torch.int32, device="cuda")
    for t, x in ((t1, x1), (t2, x2), (t1, x1)):
        ia.quantize_zp(t.cuda(), True, out=out, scales=s, zero_points=z)
        wc, ws, wz = oq.quantize_asym(x, True)
        assert np.array_equal(out.cpu().numpy(), wc)
        assert np.array_equal(s.cpu().numpy(), ws) and np.array_equal(z.cpu().numpy(), wz)
    c8, s8 = ia.quantize(t1.cuda(), True)
    w8, ws8 = oq.quantize(x1, True)
    assert np.array_equal(c8.cpu().numpy(), w8) and np.array_equal(s8.cpu().numpy(), ws8)
    assert ia.device_error() == ia.OK
