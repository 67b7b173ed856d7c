"""GPU parity of the integer GELU against the oracle: every output byte
identical, at ragged sizes, in place, with the clamp binding, over all 256
codes, and at the MLP workload's full size."""
import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl
from oracle import gelu as og

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


PARAMS = [(0.125, 0.125, 3.875), (0.04, 0.04, 4.0), (0.125, 0.0625, 3.875), (0.3, 0.35, 6.0), (0.01, 0.02, 4.5)]


def _check(ia, codes_np, p, inplace=False):
    import torch
    x = torch.from_numpy(codes_np).cuda()
    if inplace:
        y = ia.gelu(x, *p, out=x)
    else:
        y = ia.gelu(x, *p)
    got = y.cpu().numpy()
    want = og.gelu(codes_np.astype(np.int64), *p)
    if not np.array_equal(got, want):
        bad = np.flatnonzero(got.ravel() != want.ravel())
        raise AssertionError(f"{bad.size} of {got.size} differ, first at {bad[:4].tolist()}: "
                             f"got {got.ravel()[bad[:4]].tolist()} want {want.ravel()[bad[:4]].tolist()}")


@pytest.mark.parametrize("p", PARAMS)
def test_all_codes(ia, p):
    codes = np.tile(np.arange(-128, 128, dtype=np.int8), 64)  # every code in every lane position
    _check(ia, codes, p)


@pytest.mark.parametrize("n", [1, 7, 15, 16, 17, 31, 4096, 4096 * 4 + 9, 262144 + 3, 3 * 1024 * 1024 + 15])
def test_ragged_sizes(ia, n):
    rng = np.random.default_rng(n)
    _check(ia, rng.integers(-128, 128, size=n, dtype=np.int8), PARAMS[1])


@pytest.mark.parametrize("p", PARAMS[:3])
def test_in_place(ia, p):
    rng = np.random.default_rng(5)
    _check(ia, rng.integers(-128, 128, size=(333, 771), dtype=np.int8), p, inplace=True)


def test_offset_views_and_zero_length(ia):
    import torch
    rng = np.random.default_rng(9)
    base = torch.from_numpy(rng.integers(-128, 128, size=4096 + 64, dtype=np.int8)).cuda()
    x = base[16:16 + 4096]  # 16-byte aligned view
    y = ia.gelu(x, *PARAMS[0])
    assert np.array_equal(y.cpu().numpy(), og.gelu(x.cpu().numpy().astype(np.int64), *PARAMS[0]))
    with pytest.raises(ia.IntAttnError) as e:
        ia.gelu(base[3:3 + 64], *PARAMS[0])
    assert e.value.code == ia.ERR_UNSUPPORTED
    empty = torch.empty(0, dtype=torch.int8, device="cuda")
    assert ia.gelu(empty, *PARAMS[0]).numel() == 0


def test_mlp_workload_full_size(ia):
    """GPT-2-small MLP activations [16*1024, 3072] (the benchmark's size and
    launch), all 50M outputs against the oracle."""
    import torch
    spec = wl.GELU_WORKLOADS["gpt2_small_mlp_gelu_b16_l1024_f3072"]
    codes, s_x = wl.gelu_inputs_torch(spec["tokens"], spec["features"], 20251126, torch.device("cuda"))
    y = ia.gelu(codes, s_x, s_x, spec["c"])
    got = y.cpu().numpy()
    want = og.gelu(codes.cpu().numpy().astype(np.int64), s_x, s_x, spec["c"])
    assert np.array_equal(got, want)
