"""The allocation-free decode entry point, intattn_decode_static_scratch.

It serves callers that cannot allocate device memory where they call us (a
plugin living under another framework's caching allocator with no workspace
to offer, or a latency-bound loop that must not call cudaMalloc): the split-K
scratch comes from a fixed array inside the library instead of a caller
workspace.  Its output must equal intattn_decode's (which is checked against the CPU
oracle here too), call after call, while the shared array keeps whatever the
previous call left in it.

This file is collected last on purpose, so a stop-at-first-failure run has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, Lk, Lmax, d, per_head)
    (2, 3, 700, 768, 128, True),
    (4, 2, 1500, 1536, 64, False),
    (64, 32, 4096, 4096, 128, True),   # the LLaMA-7B decode shape
]


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


def _static_call(ia, x, w, out):
    import torch
    s, keep = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)._c()
    stream = torch.cuda.current_stream().cuda_stream
    rc = ia.lib().intattn_decode_static_scratch(
        x.q.data_ptr(), x.k.data_ptr(), x.v.data_ptr(), ctypes.byref(s), w.B, w.H, w.Lk, w.Lmax, w.d,
        float(w.clip_c), out.data_ptr(), stream)
    torch.cuda.synchronize()
    return rc


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Lk{}d{}".format(c[0], c[1], c[2], c[4]))
def test_static_scratch_matches_workspace_decode(ia, oracle_mod, case):
    import torch
    B, H, Lk, Lmax, d, per_head = case
    w = wl.custom_workload("noalloc", B, H, 1, Lk, d, False, per_head=per_head, clip_c=10.0,
                           index=1200 + Lk + d, decode=True, Lmax=Lmax)
    x = wl.make_inputs_torch(w, torch.device("cuda"))
    assert ia.decode_workspace_size(B, H, Lk, d) <= 48 * 1024 * 1024
    ref = ia.decode(x.q, x.k, x.v, ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=per_head), Lk, w.clip_c)
    torch.cuda.synchronize()
    want = ref.cpu().numpy()
    # the workspace decode itself against the CPU oracle, so this file stands on its own
    oracle_out = oracle_mod.decode(x.q.cpu().numpy(), x.k.cpu().numpy(), x.v.cpu().numpy(), per_head,
                                   x.s_q, x.s_k, x.s_v, x.s_o, Lk, w.clip_c)
    assert np.array_equal(want, oracle_out), f"{int((want != oracle_out).sum())} bytes differ from the oracle"
    for call in range(2):  # the second call sees the first call's leftovers
        out = torch.full_like(x.q, 99)
        rc = _static_call(ia, x, w, out)
        assert rc == ia.OK, ia.strerror(rc)
        assert ia.device_error() == ia.OK
        got = out.cpu().numpy()
        assert np.array_equal(got, want), f"call {call}: {int((got != want).sum())} bytes differ"


def test_static_scratch_rejects_oversize(ia):
    import torch
    # 4*B*H*Lk bytes of scores alone exceed the 48 MiB array; the caches are
    # real (about 0.8 GB each) so that nothing could read out of bounds even
    # if the check were missing
    B, H, Lk, d = 64, 32, 6200, 64
    assert ia.decode_workspace_size(B, H, Lk, d) > 48 * 1024 * 1024
    w = wl.custom_workload("noalloc_big", B, H, 1, Lk, d, False, clip_c=10.0, index=1300,
                           decode=True, Lmax=Lk)

    class _X:
        pass
    x = _X()
    x.q = torch.zeros((B, H, 1, d), dtype=torch.int8, device="cuda")
    x.k = torch.zeros((B, H, Lk, d), dtype=torch.int8, device="cuda")
    x.v = torch.zeros((B, H, Lk, d), dtype=torch.int8, device="cuda")
    x.s_q = x.s_k = x.s_v = x.s_o = np.array([0.05], np.float32)
    out = torch.zeros_like(x.q)
    assert _static_call(ia, x, w, out) == ia.ERR_WORKSPACE
    del x
    torch.cuda.empty_cache()
