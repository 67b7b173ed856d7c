"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function declared in include/intattn.h, derives exactly the oracle's
parameters, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ia():
    from integer_only_quantized_b200 import build
    build.build()
    import integer_only_quantized_b200 as mod
    mod.lib()
    return mod


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "intattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(intattn_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_function(ia):
    declared = _declared_functions()
    assert declared == sorted(ia.EXPORTED)
    L = ia.lib()
    for name in declared:
        assert hasattr(L, name), name
    # and the symbols are real dynamic exports of the shared object
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ia.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    for name in declared:
        assert re.search(rf"\bT {name}$", out, re.M), name


@pytest.mark.parametrize("seed", range(6))
def test_derived_params_equal_oracle(ia, oracle_mod, seed):
    rng = np.random.default_rng(seed)
    H = int(rng.integers(1, 40))
    d = int(rng.choice([64, 128]))
    per_head = bool(seed % 2)
    n = H if per_head else 1
    s_q = (10 ** rng.uniform(-3, -0.3, n)).astype(np.float32)
    s_k = (10 ** rng.uniform(-3, -0.3, n)).astype(np.float32)
    s_v = (10 ** rng.uniform(-3, 0, n)).astype(np.float32)
    s_o = (10 ** rng.uniform(-4, -1, n)).astype(np.float32)
    c = float(np.float32(rng.uniform(2, 14)))
    lut, hp = ia.derive_params(ia.Scales(s_q, s_k, s_v, s_o, per_head), H, d, c)
    olut, ohp = oracle_mod.params(per_head, s_q, s_k, s_v, s_o, H, d, c)
    assert np.array_equal(lut, olut)
    assert np.array_equal(hp, ohp)


def test_derive_params_for_the_workloads(ia, oracle_mod):
    from integer_only_quantized_b200 import workloads as wl
    for w in wl.WORKLOADS.values():
        if w.B * w.H * w.Lk * w.d > 2 ** 22:
            continue  # large inputs are covered on the GPU
        x = wl.make_inputs(w)
        sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, w.per_head)
        lut, hp = ia.derive_params(sc, w.H, w.d, w.clip_c)
        olut, ohp = oracle_mod.params(w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.H, w.d, w.clip_c)
        assert np.array_equal(lut, olut) and np.array_equal(hp, ohp), w.name


def _fwd(ia, q=1, k=1, v=1, scales=None, B=1, H=2, Lq=4, Lk=4, d=64, causal=0, c=8.0, out=1):
    sc = scales or ia.Scales(0.1, 0.1, 0.1, 0.1)
    s, keep = sc._c()
    ptr = lambda x: None if x is None else 16 * x  # aligned fake pointers, never dereferenced
    return ia.lib().intattn_forward(ptr(q), ptr(k), ptr(v), ctypes.byref(s), B, H, Lq, Lk, d, causal,
                                    c, ptr(out), None)


def test_forward_argument_errors_need_no_device(ia):
    assert _fwd(ia, d=96) == ia.ERR_UNSUPPORTED
    assert _fwd(ia, Lk=0) == ia.ERR_INVALID_ARG
    assert _fwd(ia, Lk=65536) == ia.ERR_INVALID_ARG
    assert _fwd(ia, causal=1, Lq=5, Lk=4) == ia.ERR_INVALID_ARG
    assert _fwd(ia, B=-1) == ia.ERR_INVALID_ARG
    assert _fwd(ia, H=0) == ia.ERR_INVALID_ARG
    assert _fwd(ia, c=0.0) == ia.ERR_PARAM_RANGE
    assert _fwd(ia, c=float("inf")) == ia.ERR_PARAM_RANGE
    assert _fwd(ia, scales=ia.Scales(0.0, 0.1, 0.1, 0.1)) == ia.ERR_PARAM_RANGE
    assert _fwd(ia, scales=ia.Scales(0.1, 0.1, float("nan"), 0.1)) == ia.ERR_PARAM_RANGE
    assert _fwd(ia, scales=ia.Scales(40.0, 40.0, 0.1, 0.1)) == ia.ERR_PARAM_RANGE
    assert _fwd(ia, q=None) == ia.ERR_INVALID_ARG
    assert _fwd(ia, out=None) == ia.ERR_INVALID_ARG
    too_many = ia.Scales([0.1] * 129, [0.1] * 129, [0.1] * 129, [0.1] * 129, per_head=True)
    assert _fwd(ia, H=129, scales=too_many) == ia.ERR_UNSUPPORTED
    # nothing to do: success without a launch, even with null tensors
    assert _fwd(ia, B=0, q=None, k=None, v=None, out=None) == ia.OK
    assert _fwd(ia, Lq=0, q=None, out=None) == ia.OK
    # a scale-less call
    L = ia.lib()
    assert L.intattn_forward(16, 16, 16, None, 1, 1, 4, 4, 64, 0, 8.0, 16, None) == ia.ERR_INVALID_ARG


def test_forward_variant_argument_errors_need_no_device(ia):
    sc = ia.Scales(0.1, 0.1, 0.1, 0.1)
    s, keep = sc._c()
    L = ia.lib()

    def fv(variant, Lk=4, d=64, B=1):
        return L.intattn_forward_variant(16, 16, 16, ctypes.byref(s), B, 2, 4, Lk, d, 0, 8.0, 16, variant, None)

    assert fv(3) == ia.ERR_INVALID_ARG
    assert fv(-1) == ia.ERR_INVALID_ARG
    assert fv(ia.VARIANT_SHORT_ROWS, Lk=ia.SHORT_ROWS_MAX_KEYS + 1) == ia.ERR_UNSUPPORTED
    assert fv(ia.VARIANT_THREE_PASS, d=96) == ia.ERR_UNSUPPORTED
    assert fv(ia.VARIANT_SHORT_ROWS, Lk=0) == ia.ERR_INVALID_ARG
    for variant in (ia.VARIANT_AUTO, ia.VARIANT_THREE_PASS, ia.VARIANT_SHORT_ROWS):
        assert fv(variant, B=0) == ia.OK  # nothing to do, no launch


def test_forward_fp_argument_errors_need_no_device(ia):
    import numpy as np
    L = ia.lib()
    f32p = ctypes.POINTER(ctypes.c_float)
    so = np.array([0.03, 0.03], np.float32)
    bad = np.array([0.03, 0.0], np.float32)
    need = ia.forward_fp_workspace_size(1, 2, 64, 64, 64)
    assert need > 3 * 2 * 64 * 64 and ia.forward_fp_workspace_size(1, 2, 64, 64, 96) == 0

    def call(dtype=1, per_head=1, s_o=so, d=64, ws=256, wsb=None, B=1):
        return L.intattn_forward_fp(16, 16, 16, dtype, per_head, s_o.ctypes.data_as(f32p) if s_o is not None else None,
                                    None, 8.0, B, 2, 64, 64, d, 0, 16, None, ws,
                                    need if wsb is None else wsb, None)

    assert call(dtype=7) == ia.ERR_UNSUPPORTED
    assert call(d=96) == ia.ERR_UNSUPPORTED
    assert call(s_o=None) == ia.ERR_INVALID_ARG
    assert call(s_o=bad) == ia.ERR_PARAM_RANGE
    assert call(wsb=need - 1) == ia.ERR_WORKSPACE
    assert call(ws=None) == ia.ERR_WORKSPACE
    assert call(ws=256 + 16) == ia.ERR_WORKSPACE   # misaligned workspace
    assert call(B=0) == ia.OK                        # nothing to do, no launch


def test_quantize_zp_argument_errors_need_no_device(ia):
    L = ia.lib()

    def call(dtype=1, B=1, H=2, Lr=64, d=64, x=16, out=16, scales=256, zps=512):
        return L.intattn_quantize_zp(x, dtype, B, H, Lr, d, 1, out, scales, zps, None)

    assert call(zps=None) == ia.ERR_INVALID_ARG
    assert call(scales=None) == ia.ERR_INVALID_ARG
    assert call(dtype=5) == ia.ERR_UNSUPPORTED
    assert call(Lr=3, d=6) == ia.ERR_UNSUPPORTED      # L * d not whole 16-byte vectors
    assert call(zps=514) == ia.ERR_UNSUPPORTED        # misaligned zero-point buffer
    assert call(H=0) == ia.ERR_INVALID_ARG
    assert call(x=None) == ia.ERR_INVALID_ARG
    assert call(out=24) == ia.ERR_UNSUPPORTED         # misaligned codes


def test_zero_point_argument_errors_need_no_device(ia):
    """Zero-points out of 0..255 (0..15 for int4 codes) are rejected before
    any launch; the calibration takes no zero-points."""
    import numpy as np
    L = ia.lib()
    one = np.array([0.02], np.float32)

    def scales(zk=None, zv=None):
        return ia.Scales(one, one, one, one, z_k=zk, z_v=zv)._c()

    for zk, zv in ((256, None), (None, -1), (0, 300)):
        sc, keep = scales(zk, zv)
        rc = L.intattn_forward_variant(16, 16, 16, ctypes.byref(sc), 1, 2, 64, 64, 64, 0, 8.0, 16, 0, None)
        assert rc == ia.ERR_INVALID_ARG, (zk, zv)
        rc = L.intattn_decode(16, 16, 16, ctypes.byref(sc), 1, 2, 64, 64, 64, 8.0, 16, 256, 1 << 20, None)
        assert rc == ia.ERR_INVALID_ARG, (zk, zv)
    for zk, zv in ((16, None), (None, 16), (-1, 3)):  # unsigned int4 codes: zero-points 0 .. 15
        sc, keep = scales(zk, zv)
        assert L.intattn_decode_int4(16, 16, 16, ctypes.byref(sc), 1, 2, 64, 64, 64, 8.0, 16, 256, 1 << 20,
                                     None) == ia.ERR_INVALID_ARG
    sc, keep = scales(3, 4)
    clip = np.zeros(1, np.float32)
    assert L.intattn_calibrate_clip(16, 16, ctypes.byref(sc), 1, 2, 64, 64, 64, 0, 4, 4, 0.5, 8.0,
                                    clip.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), None, 256, 1 << 20,
                                    None) == ia.ERR_UNSUPPORTED


def test_calibrate_argument_errors_need_no_device(ia):
    import numpy as np
    L = ia.lib()
    sc = ia.Scales([0.02, 0.03], [0.02, 0.03], [0.1, 0.1], [0.1, 0.1], per_head=True)
    s, keep_alive = sc._c()
    clip = np.zeros(2, np.float32)
    fp = ctypes.POINTER(ctypes.c_float)
    ws = ia.lib().intattn_calibrate_workspace_size(1, 2)
    assert ws >= 8 and ia.lib().intattn_calibrate_workspace_size(1, 0) == 0

    def call(keep=4, stride=2, c_min=0.5, c_max=20.0, out=True, d=64, wsb=None, B=1):
        return L.intattn_calibrate_clip(16, 16, ctypes.byref(s), B, 2, 64, 64, d, 0, keep, stride, c_min, c_max,
                                        clip.ctypes.data_as(fp) if out else None, None, 256,
                                        ws if wsb is None else wsb, None)

    assert call(keep=0) == ia.ERR_INVALID_ARG
    assert call(stride=0) == ia.ERR_INVALID_ARG
    assert call(c_min=0.0) == ia.ERR_PARAM_RANGE
    assert call(c_max=0.1) == ia.ERR_PARAM_RANGE
    assert call(out=False) == ia.ERR_INVALID_ARG
    assert call(d=96) == ia.ERR_UNSUPPORTED
    assert call(wsb=ws - 4) == ia.ERR_WORKSPACE
    # nothing sampled (B = 0): no launch, every threshold is c_min
    assert call(B=0, c_min=0.75) == ia.OK and clip.tolist() == [0.75, 0.75]


def test_misaligned_pointer_is_rejected(ia):
    sc = ia.Scales(0.1, 0.1, 0.1, 0.1)
    s, keep = sc._c()
    L = ia.lib()
    assert L.intattn_forward(16 * 5 + 8, 16, 16, ctypes.byref(s), 1, 1, 4, 4, 64, 0, 8.0, 16,
                             None) == ia.ERR_UNSUPPORTED


def test_decode_argument_errors_need_no_device(ia):
    sc = ia.Scales(0.1, 0.1, 0.1, 0.1)
    s, keep = sc._c()
    L = ia.lib()
    ws = ia.decode_workspace_size(2, 3, 700, 128)
    assert ws > 2 * 3 * 700 * 4
    assert ia.decode_workspace_size(2, 3, 0, 128) == 0
    assert ia.decode_workspace_size(2, 3, 700, 96) == 0
    args = lambda **kw: dict(dict(q=16, k=16, v=16, B=2, H=3, Lk=700, Lmax=768, d=128, c=8.0, out=16,
                                  ws=256, wsb=ws), **kw)

    def call(**kw):
        a = args(**kw)
        return L.intattn_decode(a["q"], a["k"], a["v"], ctypes.byref(s), a["B"], a["H"], a["Lk"],
                                a["Lmax"], a["d"], a["c"], a["out"], a["ws"], a["wsb"], None)
    assert call(Lmax=600) == ia.ERR_INVALID_ARG
    assert call(d=32) == ia.ERR_UNSUPPORTED
    assert call(wsb=ws - 1) == ia.ERR_WORKSPACE
    assert call(ws=None) == ia.ERR_WORKSPACE
    assert call(ws=256 + 16) == ia.ERR_WORKSPACE
    assert call(k=None) == ia.ERR_INVALID_ARG
    assert call(B=0, q=None) == ia.OK


def test_strerror(ia):
    for code in range(7):
        assert ia.strerror(code)
    assert "unknown" in ia.strerror(99)


def test_binding_rejects_cpu_tensors(ia):
    import torch
    x = torch.zeros(1, 1, 4, 64, dtype=torch.int8)
    with pytest.raises(TypeError):
        ia.forward(x, x, x, ia.Scales(0.1, 0.1, 0.1, 0.1), False, 8.0)


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch, ia):
    import integer_only_quantized_b200 as mod
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        mod.lib()


def test_forward_host_checks_without_gpu():
    """Argument checks of intattn_forward_host return before any CUDA call."""
    import ctypes
    import integer_only_quantized_b200 as ia
    L = ia.lib()
    one = np.ones(1, dtype=np.float32)
    sc = ia.Scales(one, one, one, one)
    c, keep = sc._c()
    f = L.intattn_forward_host
    need = L.intattn_forward_host_workspace_size(2, 3, 64, 64, 64)
    assert need > 0 and need % 256 == 0
    assert L.intattn_forward_host_workspace_size(2, 3, 64, 64, 96) == 0
    args = lambda B, ws, nbytes: (16, 16, 16, ctypes.byref(c), B, 3, 64, 64, 64, 0, 8.0, 16, ws, nbytes, None)
    assert f(*args(-1, 256, need)) == ia.ERR_INVALID_ARG
    assert f(*args(0, 256, need)) == ia.OK                 # nothing to do
    assert f(*args(2, 256, need - 1)) == ia.ERR_WORKSPACE
    assert f(*args(2, 0, need)) == ia.ERR_WORKSPACE
    assert f(*args(2, 256 + 16, need)) == ia.ERR_WORKSPACE  # not 256-byte aligned
    del keep
