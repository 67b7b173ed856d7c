"""Per-head clip thresholds: host parameter derivation (no device)."""
import ctypes

import numpy as np
import pytest


@pytest.fixture(scope="module")
def ia():
    from integer_only_quantized_b200 import build
    build.build()
    import integer_only_quantized_b200 as mod
    mod.lib()
    return mod


def test_per_head_clip_params_equal_oracle_per_head(ia, oracle_mod):
    H = 5
    rng = np.random.default_rng(8)
    s = [rng.uniform(0.005, 0.05, H).astype(np.float32) for _ in range(4)]
    clips = np.array([4.0, 6.0, 10.0, 6.0, 12.5], np.float32)
    lut, hp = ia.derive_params(ia.Scales(*s, per_head=True, clip=clips), H, 128, 99.0)
    for h in range(H):
        L, want = oracle_mod.params(True, s[0][h:h + 1], s[1][h:h + 1], s[2][h:h + 1], s[3][h:h + 1], 1, 128,
                                    float(clips[h]))
        assert hp[h].tolist() == want[0].tolist(), h
    # the returned table is head 0's
    assert lut.tolist() == oracle_mod.lut(float(clips[0])).tolist()


def test_no_clip_array_means_the_call_argument(ia):
    s = [np.full(3, 0.02, np.float32)] * 4
    a = ia.derive_params(ia.Scales(*s, per_head=True), 3, 64, 7.0)
    b = ia.derive_params(ia.Scales(*s, per_head=True, clip=np.full(3, 7.0, np.float32)), 3, 64, 1.0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_too_many_distinct_clips_is_unsupported(ia):
    H = ia.MAX_CLIPS + 1
    s = [np.full(H, 0.02, np.float32)] * 4
    with pytest.raises(ia.IntAttnError) as e:
        ia.derive_params(ia.Scales(*s, per_head=True, clip=np.arange(1, H + 1, dtype=np.float32)), H, 64, 8.0)
    assert e.value.code == ia.ERR_UNSUPPORTED
    # the same count of heads with repeated values is fine
    ia.derive_params(ia.Scales(*s, per_head=True, clip=np.tile(np.float32([4, 8]), H)[:H]), H, 64, 8.0)


def test_bad_per_head_clip_is_param_range(ia):
    s = [np.full(2, 0.02, np.float32)] * 4
    with pytest.raises(ia.IntAttnError) as e:
        ia.derive_params(ia.Scales(*s, per_head=True, clip=np.float32([8.0, -1.0])), 2, 64, 8.0)
    assert e.value.code == ia.ERR_PARAM_RANGE
