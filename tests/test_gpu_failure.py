"""Failure detection on the GPU without a fault: a kernel wait that can never
complete gives up after its time limit, the host reads INTATTN_ERR_TIMEOUT,
and the context keeps working."""
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


def test_bounded_wait_reports_timeout_and_context_survives(ia, oracle_mod):
    import torch
    assert ia.device_error() == ia.OK
    assert ia.selftest_timeout() == ia.ERR_TIMEOUT
    assert ia.device_error() == ia.OK  # the word was cleared by the read
    # the same context still computes correct results
    w = wl.custom_workload("after_timeout", 1, 2, 130, 130, 64, True, index=1400)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o)
    out = ia.forward(*(torch.from_numpy(a).cuda() for a in (x.q, x.k, x.v)), sc, True, w.clip_c)
    assert ia.device_error() == ia.OK
    want = oracle_mod.forward(x.q, x.k, x.v, False, x.s_q, x.s_k, x.s_v, x.s_o, True, w.clip_c)
    assert np.array_equal(out.cpu().numpy(), want)
