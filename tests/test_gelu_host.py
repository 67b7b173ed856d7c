"""Host side of the integer GELU, without a GPU: the library's parameter
derivation equals the oracle's, and intattn_gelu's argument checks return
their documented codes before anything is launched."""
import numpy as np
import pytest

import integer_only_quantized_b200 as ia
from oracle import gelu as og


@pytest.fixture(scope="module")
def lib():
    from integer_only_quantized_b200 import build
    build.build()
    return ia.lib()


def _cases(n, seed):
    rng = np.random.default_rng(seed)
    fixed = [(0.125, 0.125, 3.875), (0.04, 0.04, 4.0), (5.0 / 127, 6.0 / 127, 3.0), (1.0, 1.0, 0.5),
             (1e-3, 1e-3, 8.0), (0.3, 0.01, 6.0)]
    rand = [(10 ** rng.uniform(-4, 1), 10 ** rng.uniform(-4, 1), rng.uniform(0.25, 10.0)) for _ in range(n)]
    return fixed + rand


def test_params_match_oracle(lib):
    for s_x, s_y, c in _cases(2000, 7):
        try:
            want = og.gelu_params(s_x, s_y, c)
        except og.ParamRange:
            with pytest.raises(ia.IntAttnError) as e:
                ia.gelu_params(s_x, s_y, c)
            assert e.value.code == ia.ERR_PARAM_RANGE
            continue
        M, s, G, Mo, so = ia.gelu_params(s_x, s_y, c)
        assert (M, s, G, Mo, so) == (want[0], want[1], list(want[2]), want[3], want[4]), (s_x, s_y, c)


@pytest.mark.parametrize("args", [(0.0, 0.1, 4.0), (0.1, -1.0, 4.0), (0.1, 0.1, 0.0), (float("inf"), 0.1, 4.0),
                                  (0.1, 0.1, float("nan")), (1e-12, 0.1, 1e6), (1e-10, 1e3, 4.0), (1e30, 1.0, 1e-3)])
def test_param_range(lib, args):
    p = ia._GeluParams()
    import ctypes
    assert lib.intattn_gelu_derive_params(*[float(a) for a in args], ctypes.byref(p)) == ia.ERR_PARAM_RANGE
    assert lib.intattn_gelu(16, 32, 64, *[float(a) for a in args], None) == ia.ERR_PARAM_RANGE


def test_argument_checks(lib):
    g = lib.intattn_gelu
    ok = (0.05, 0.05, 4.0)
    assert lib.intattn_gelu_derive_params(*ok, None) == ia.ERR_INVALID_ARG
    assert g(16, 32, -1, *ok, None) == ia.ERR_INVALID_ARG
    assert g(0, 0, 0, *ok, None) == ia.OK            # nothing to do, nothing launched
    assert g(0, 4096, 64, *ok, None) == ia.ERR_INVALID_ARG
    assert g(4096, 0, 64, *ok, None) == ia.ERR_INVALID_ARG
    assert g(4096 + 8, 8192, 64, *ok, None) == ia.ERR_UNSUPPORTED
    assert g(4096, 8192 + 4, 64, *ok, None) == ia.ERR_UNSUPPORTED
    assert g(4096, 4096 + 32, 64, *ok, None) == ia.ERR_INVALID_ARG   # partial overlap
    assert g(4096 + 32, 4096, 64, *ok, None) == ia.ERR_INVALID_ARG


def test_gelu_workload_recipe():
    """Input generator shares no arithmetic with the method: it only draws
    codes; check the shape of what it draws on the CPU."""
    import torch
    from integer_only_quantized_b200 import workloads as wl
    codes, s_x = wl.gelu_inputs_torch(64, 768, 3, torch.device("cpu"))
    assert codes.dtype == torch.int8 and codes.shape == (64, 768)
    assert int(codes.abs().max()) == 127 and s_x > 0
