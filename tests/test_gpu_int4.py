"""GPU parity of the int4-KV decode: the packed-nibble kernels against the
CPU oracle run on the unpacked codes (the same integer definition with K and
V codes in [-8, 7]), byte for byte."""
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


def _assert_equal(got, want, what):
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{what}: {len(bad)} of {got.size} bytes differ; first at {bad[:5].tolist()} "
                             f"got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")


SWEEP = [
    (1, 1, 1, 1, 64), (2, 3, 100, 160, 128), (1, 2, 511, 511, 64), (1, 2, 512, 512, 128),
    (2, 2, 513, 600, 64), (3, 2, 1500, 2048, 128), (1, 4, 4096, 4100, 64), (1, 2, 4097, 4097, 128),
    (2, 1, 9000, 9000, 128),
]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "B{}H{}Lk{}Lmax{}d{}".format(*c))
def test_decode_int4_sweep_full_code_range(ia, oracle_mod, case):
    """Uniform codes over all of [-8, 7] (the extremes included)."""
    import torch
    B, H, Lk, Lmax, d = case
    w = wl.custom_workload("dec4", B, H, 1, Lk, d, False, per_head=True, clip_c=10.0,
                           index=600 + Lk + d, decode=True, Lmax=Lmax, kv_bits=4)
    x = wl.make_inputs(w)
    rng = np.random.default_rng(w.seed)
    k = rng.integers(-8, 8, size=x.k.shape).astype(np.int8)
    v = rng.integers(-8, 8, size=x.v.shape).astype(np.int8)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True)
    ws = torch.randint(0, 255, (ia.decode_workspace_size(B, H, Lk, d),), dtype=torch.uint8, device="cuda")
    out = ia.decode_int4(_dev(x.q), _dev(wl.pack_int4(k)), _dev(wl.pack_int4(v)), sc, Lk, w.clip_c,
                         workspace=ws)
    assert ia.device_error() == ia.OK
    want = oracle_mod.decode(x.q, k, v, True, x.s_q, x.s_k, x.s_v, x.s_o, Lk, w.clip_c)
    _assert_equal(out.cpu().numpy(), want, str(case))


def test_decode_int4_workload_full(ia, oracle_mod):
    """The LLaMA-7B int4 decode workload, every output byte."""
    w = wl.WORKLOADS["llama7b_decode_int4_b64_lk4096"]
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    out = ia.decode_int4(_dev(x.q), _dev(wl.pack_int4(x.k)), _dev(wl.pack_int4(x.v)), sc, w.Lk, w.clip_c)
    assert ia.device_error() == ia.OK
    want = oracle_mod.decode(x.q, x.k, x.v, w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.Lk, w.clip_c)
    _assert_equal(out.cpu().numpy(), want, w.name)


def test_decode_int4_equals_int8_decode_of_the_same_codes(ia):
    """Two independent kernels over the same codes (int8 storage vs packed)."""
    w = wl.custom_workload("dec4x8", 3, 4, 1, 2000, 128, False, per_head=False, clip_c=8.0, index=77,
                           decode=True, Lmax=2048, kv_bits=4)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=False)
    a = ia.decode_int4(_dev(x.q), _dev(wl.pack_int4(x.k)), _dev(wl.pack_int4(x.v)), sc, w.Lk, w.clip_c)
    b = ia.decode(_dev(x.q), _dev(x.k), _dev(x.v), sc, w.Lk, w.clip_c)
    assert ia.device_error() == ia.OK
    _assert_equal(a.cpu().numpy(), b.cpu().numpy(), "int4 vs int8 storage")
