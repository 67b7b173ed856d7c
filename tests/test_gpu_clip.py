"""GPU parity with per-head clip thresholds: every head is the scalar
definition with its own threshold, so the oracle runs head by head."""
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


def _oracle_per_head(fn, x, clips, **kw):
    outs = []
    for h in range(len(clips)):
        sl = slice(h, h + 1)
        outs.append(fn(x.q[:, sl], x.k[:, sl], x.v[:, sl], True, x.s_q[sl], x.s_k[sl], x.s_v[sl], x.s_o[sl],
                       clip_c=float(clips[h]), **kw))
    return np.concatenate(outs, axis=1)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_forward_per_head_clip(ia, oracle_mod, d, causal):
    w = wl.custom_workload("clip_h", 2, 4, 300, 300, d, causal, per_head=True, clip_c=8.0, index=970 + d)
    x = wl.make_inputs(w)
    clips = np.float32([3.0, 6.0, 10.0, 6.0])
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True, clip=clips)
    out = ia.forward(_dev(x.q), _dev(x.k), _dev(x.v), sc, causal, 99.0).cpu().numpy()
    assert ia.device_error() == ia.OK
    want = _oracle_per_head(lambda q, k, v, ph, sq, sk, sv, so, clip_c: oracle_mod.forward(
        q, k, v, ph, sq, sk, sv, so, causal, clip_c), x, clips)
    assert np.array_equal(out, want)


@pytest.mark.parametrize("kv_bits", [8, 4])
def test_decode_per_head_clip(ia, oracle_mod, kv_bits):
    w = wl.custom_workload("clip_dec", 3, 4, 1, 1500, 128, False, per_head=True, clip_c=10.0, index=990 + kv_bits,
                           decode=True, Lmax=1600, kv_bits=kv_bits)
    x = wl.make_inputs(w)
    clips = np.float32([5.0, 10.0, 14.0, 5.0])
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True, clip=clips)
    if kv_bits == 4:
        out = ia.decode_int4(_dev(x.q), _dev(wl.pack_int4(x.k)), _dev(wl.pack_int4(x.v)), sc, w.Lk, 99.0)
    else:
        out = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, w.Lk, 99.0)
    assert ia.device_error() == ia.OK
    want = _oracle_per_head(lambda q, k, v, ph, sq, sk, sv, so, clip_c: oracle_mod.decode(
        q, k, v, ph, sq, sk, sv, so, w.Lk, clip_c), x, clips)
    assert np.array_equal(out.cpu().numpy(), want)
