"""Adaptive clip thresholds on the GPU (intattn_calibrate_clip) against the
CPU oracle (oracle/calibrate.py): the integer gaps must be equal, and so the
thresholds (the same double formula on the host).  Then the thresholds in
use: a forward with the calibrated per-head clips equals the oracle run head
by head with them."""
import numpy as np
import pytest

from integer_only_quantized_b200 import workloads as wl
from oracle import calibrate as oc

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


CASES = [  # B, H, Lq, Lk, d, causal, per_head, keep, stride
    (2, 3, 200, 200, 64, False, True, 8, 4),
    (1, 2, 300, 700, 128, True, True, 16, 7),
    (2, 2, 129, 129, 64, True, False, 1, 1),
    (1, 3, 50, 50, 128, True, True, 64, 3),     # keep larger than the early causal rows
    (1, 2, 40, 40, 64, False, True, 5, 64),     # stride beyond Lq: no sampled row, c = c_min
    (2, 3, 517, 517, 128, True, True, 20, 5),   # 103 sampled rows: shared-memory kernel, ragged last CTA
    (1, 1, 52000, 52000, 64, True, True, 8, 5200),  # rows too long for shared memory: the recomputing kernel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}k{}s{}".format(
    *c[:5], "c" if c[5] else "", "h" if c[6] else "", c[7], c[8]))
def test_calibrate_matches_oracle(ia, case):
    B, H, Lq, Lk, d, causal, per_head, keep, stride = case
    w = wl.custom_workload("calib", B, H, Lq, Lk, d, causal, per_head=per_head, index=4000 + Lq + Lk + keep)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=per_head)
    clip, gaps = ia.calibrate_clip(_dev(x.q), _dev(x.k), sc, causal, keep, stride, c_min=0.5, c_max=40.0)
    want_c, want_g = oc.thresholds(x.q, x.k, per_head, x.s_q, x.s_k, causal, keep, stride, 0.5, 40.0)
    assert np.array_equal(gaps, want_g.astype(np.int32)), (gaps, want_g)
    assert np.array_equal(clip, want_c), (clip, want_c)


@pytest.mark.parametrize("name,keep,stride", [("vit_b16_l197", 16, 3), ("gpt2_small_causal_l2048", 32, 31)])
def test_calibrate_workloads(ia, name, keep, stride):
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    clip, gaps = ia.calibrate_clip(_dev(x.q), _dev(x.k), sc, w.causal, keep, stride)
    want_c, want_g = oc.thresholds(x.q, x.k, w.per_head, x.s_q, x.s_k, w.causal, keep, stride, 0.25, 64.0)
    assert np.array_equal(gaps, want_g.astype(np.int32))
    assert np.array_equal(clip, want_c)


def test_calibrated_clips_in_the_forward(ia, oracle_mod):
    """Per-head thresholds from calibration (at most 8 distinct per call)
    drive the forward; each head equals the oracle with its own threshold."""
    B, H, L, d = 1, 6, 256, 64
    w = wl.custom_workload("calib_fwd", B, H, L, L, d, True, per_head=True, index=4100)
    x = wl.make_inputs(w)
    q, k, v = _dev(x.q), _dev(x.k), _dev(x.v)
    clip, _ = ia.calibrate_clip(q, k, ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True), True, 12, 8)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True, clip=clip)
    got = ia.forward(q, k, v, sc, True, 8.0).cpu().numpy()
    assert ia.device_error() == ia.OK
    for h in range(H):
        want = oracle_mod.forward(x.q[:, h:h + 1], x.k[:, h:h + 1], x.v[:, h:h + 1], True, x.s_q[h:h + 1],
                                  x.s_k[h:h + 1], x.s_v[h:h + 1], x.s_o[h:h + 1], True, float(clip[h]))
        assert np.array_equal(got[:, h:h + 1], want), f"head {h}"
