"""int4 KV cache: byte layout of the packing and the C ABI's argument checks
(no device needed)."""
import ctypes

import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl


def test_pack_layout_hand_example():
    # channels (1, -1, 7, -8): byte 0 = 0xF1 (channel 1 = -1 = 0xF in the high
    # nibble, channel 0 = 1 in the low nibble), byte 1 = 0x87
    codes = np.array([[1, -1, 7, -8]], dtype=np.int8)
    assert wl.pack_int4(codes).tolist() == [[0xF1, 0x87]]
    assert wl.unpack_int4(np.array([[0xF1, 0x87]], dtype=np.uint8)).tolist() == [[1, -1, 7, -8]]


def test_pack_round_trip_every_pair():
    a, b = np.meshgrid(np.arange(-8, 8), np.arange(-8, 8), indexing="ij")
    codes = np.stack([a.ravel(), b.ravel()], axis=1).astype(np.int8)  # all 256 channel pairs
    packed = wl.pack_int4(codes)
    assert sorted(packed.ravel().tolist()) == list(range(256))  # a bijection onto bytes
    assert np.array_equal(wl.unpack_int4(packed), codes)


def test_pack_rejects_out_of_range_and_odd_width():
    with pytest.raises(ValueError):
        wl.pack_int4(np.array([[8, 0]], dtype=np.int8))
    with pytest.raises(ValueError):
        wl.pack_int4(np.array([[0, 0, 0]], dtype=np.int8))


def test_int4_workload_codes_and_bytes():
    w = wl.custom_workload("i4", 2, 2, 1, 300, 64, False, per_head=True, clip_c=10.0, index=40,
                           decode=True, Lmax=320, kv_bits=4)
    x = wl.make_inputs(w)
    assert x.k.min() >= -7 and x.k.max() <= 7 and x.v.min() >= -7 and x.v.max() <= 7
    assert x.q.min() >= -127  # q stays int8
    assert w.decode_bytes == 2 * 2 * 2 * 300 * 64 // 2 + 2 * 2 * 2 * 64


@pytest.fixture(scope="module")
def ia():
    from integer_only_quantized_b200 import build
    build.build()
    import integer_only_quantized_b200 as mod
    mod.lib()
    return mod


def test_decode_int4_argument_errors_need_no_device(ia):
    sc = ia.Scales(0.1, 0.1, 0.1, 0.1)
    s, keep = sc._c()
    L = ia.lib()
    ws = ia.decode_workspace_size(2, 3, 700, 128)

    def call(**kw):
        a = dict(dict(q=16, k=16, v=16, B=2, H=3, Lk=700, Lmax=768, d=128, c=8.0, out=16, ws=256, wsb=ws), **kw)
        return L.intattn_decode_int4(a["q"], a["k"], a["v"], ctypes.byref(s), a["B"], a["H"], a["Lk"],
                                     a["Lmax"], a["d"], a["c"], a["out"], a["ws"], a["wsb"], None)
    assert call(Lmax=600) == ia.ERR_INVALID_ARG
    assert call(d=96) == ia.ERR_UNSUPPORTED
    assert call(k=24) == ia.ERR_UNSUPPORTED          # not 16-byte aligned
    assert call(wsb=ws - 1) == ia.ERR_WORKSPACE
    assert call(v=None) == ia.ERR_INVALID_ARG
    assert call(c=-1.0) == ia.ERR_PARAM_RANGE
    assert call(B=0, q=None) == ia.OK
