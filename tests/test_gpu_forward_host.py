"""The forward from host buffers (intattn_forward_host): copies in, forward,
copy out, with consecutive calls alternating between two workspace slots so
that they overlap.  Its output must be identical to the device forward's
(itself byte-identical to the oracle) and to the oracle: per-head scales and
thresholds, causal masks, pinned and pageable host memory, and a run of
overlapping calls on distinct inputs."""
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


def _host(a, pinned):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.pin_memory() if pinned else t


CASES = [  # B, H, Lq, Lk, d, causal, per_head, pinned
    (8, 12, 128, 128, 64, False, False, True),
    (11, 3, 70, 200, 64, True, True, True),
    (1, 12, 300, 300, 64, False, True, True),
    (3, 5, 129, 257, 128, True, True, False),     # pageable memory
    (2, 32, 64, 513, 128, False, False, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}Lq{}Lk{}d{}{}{}{}".format(
    *c[:5], "c" if c[5] else "", "h" if c[6] else "", "p" if c[7] else ""))
def test_forward_host_matches_oracle(ia, oracle_mod, case):
    import torch
    B, H, Lq, Lk, d, causal, per_head, pinned = case
    w = wl.custom_workload("host", B, H, Lq, Lk, d, causal, per_head=per_head, index=1100 + B * 7 + H)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=per_head)
    q, k, v = (_host(a, pinned) for a in (x.q, x.k, x.v))
    out = torch.full(x.q.shape, 0x5A, dtype=torch.int8)
    out = out.pin_memory() if pinned else out
    ia.forward_host(q, k, v, sc, causal, w.clip_c, out=out)
    torch.cuda.synchronize()
    assert ia.device_error() == ia.OK
    want = oracle_mod.forward(x.q, x.k, x.v, per_head, x.s_q, x.s_k, x.s_v, x.s_o, causal, w.clip_c)
    assert np.array_equal(out.numpy(), want)


def test_forward_host_per_head_clip_and_reuse(ia, oracle_mod):
    """Per-head thresholds follow the chunk's heads; a second call into the
    same workspace and output gives the same bytes."""
    import torch
    w = wl.custom_workload("host_clip", 1, 8, 200, 200, 64, True, per_head=True, clip_c=8.0, index=1200)
    x = wl.make_inputs(w)
    clips = np.array([4.0, 5.0, 6.0, 7.0, 8.0, 9.0, 10.0, 12.0], dtype=np.float32)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True, clip=clips)
    q, k, v = (_host(a, True) for a in (x.q, x.k, x.v))
    ws = torch.empty(ia.forward_host_workspace_size(1, 8, 200, 200, 64), dtype=torch.uint8, device="cuda")
    out = torch.empty(x.q.shape, dtype=torch.int8).pin_memory()
    want = np.concatenate([oracle_mod.forward(x.q[:, h:h + 1], x.k[:, h:h + 1], x.v[:, h:h + 1], True,
                                              x.s_q[h:h + 1], x.s_k[h:h + 1], x.s_v[h:h + 1], x.s_o[h:h + 1],
                                              True, float(clips[h])) for h in range(8)], axis=1)
    for _ in range(2):
        ia.forward_host(q, k, v, sc, True, 8.0, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(out.numpy(), want)


def test_forward_host_overlapping_calls(ia, oracle_mod):
    """Six calls in a row on one stream and one workspace (the slots
    alternate, each call's copies in overlap the previous forward), each on
    its own inputs and into its own output; every output checked after one
    synchronisation."""
    import torch
    runs = []
    for i in range(6):
        w = wl.custom_workload("host_seq", 2, 4, 160, 160, 64, bool(i % 2), per_head=True, index=1300 + i)
        x = wl.make_inputs(w)
        runs.append((w, x, [_host(a, True) for a in (x.q, x.k, x.v)],
                     torch.empty(x.q.shape, dtype=torch.int8).pin_memory()))
    ws = torch.empty(ia.forward_host_workspace_size(2, 4, 160, 160, 64), dtype=torch.uint8, device="cuda")
    for w, x, (q, k, v), out in runs:
        ia.forward_host(q, k, v, ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True), w.causal, w.clip_c,
                        out=out, workspace=ws)
    torch.cuda.synchronize()
    for w, x, _, out in runs:
        want = oracle_mod.forward(x.q, x.k, x.v, True, x.s_q, x.s_k, x.s_v, x.s_o, w.causal, w.clip_c)
        assert np.array_equal(out.numpy(), want)


def test_forward_host_two_workspaces_two_streams(ia, oracle_mod):
    """Calls alternating between two workspaces, each on its own stream:
    every workspace keeps its own slot order, so no call overwrites a slot
    that the other stream's forward still reads."""
    import torch
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(ia.forward_host_workspace_size(2, 4, 192, 192, 64), dtype=torch.uint8, device="cuda")
           for _ in range(2)]
    runs = []
    for i in range(8):
        w = wl.custom_workload("host_two", 2, 4, 192, 192, 64, bool(i % 3 == 0), per_head=bool(i % 2),
                               index=1400 + i)
        x = wl.make_inputs(w)
        runs.append((w, x, [_host(a, True) for a in (x.q, x.k, x.v)],
                     torch.empty(x.q.shape, dtype=torch.int8).pin_memory()))
    for i, (w, x, (q, k, v), out) in enumerate(runs):
        ia.forward_host(q, k, v, ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head), w.causal,
                        w.clip_c, out=out, workspace=wss[i % 2], stream=streams[i % 2])
    torch.cuda.synchronize()
    for w, x, _, out in runs:
        want = oracle_mod.forward(x.q, x.k, x.v, w.per_head, x.s_q, x.s_k, x.s_v, x.s_o, w.causal, w.clip_c)
        assert np.array_equal(out.numpy(), want)


def test_forward_host_matches_device_forward_on_bench_workload(ia):
    """BERT-base B8 H12 L512: host path == device path, byte for byte."""
    import torch
    w = wl.WORKLOADS["bert_base_b8_l512"]
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=w.per_head)
    dev = ia.forward(*(torch.from_numpy(a).cuda() for a in (x.q, x.k, x.v)), sc, w.causal, w.clip_c)
    host = ia.forward_host(*(_host(a, True) for a in (x.q, x.k, x.v)), sc, w.causal, w.clip_c)
    torch.cuda.synchronize()
    assert np.array_equal(host.numpy(), dev.cpu().numpy())


def test_forward_host_workspace_errors(ia):
    import torch
    w = wl.custom_workload("host_ws", 2, 2, 64, 64, 64, False, index=1210)
    x = wl.make_inputs(w)
    sc = ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o)
    q, k, v = (_host(a, True) for a in (x.q, x.k, x.v))
    small = torch.empty(ia.forward_host_workspace_size(2, 2, 64, 64, 64) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ia.IntAttnError) as e:
        ia.forward_host(q, k, v, sc, False, w.clip_c, workspace=small)
    assert e.value.code == ia.ERR_WORKSPACE


def test_forward_host_under_stream_capture(ia, oracle_mod):
    """Uncaptured calls first (their slot events are recorded outside any
    capture), then two calls captured as a CUDA graph on the same workspace
    and replayed twice, then uncaptured calls again: every output equals the
    oracle's.  A captured call must not wait on events recorded outside the
    capture, nor an uncaptured call on events recorded inside one."""
    import torch
    runs = []
    for i in range(2):
        w = wl.custom_workload("host_graph", 2, 3, 150, 150, 64, bool(i), per_head=True, index=1500 + i)
        x = wl.make_inputs(w)
        want = oracle_mod.forward(x.q, x.k, x.v, True, x.s_q, x.s_k, x.s_v, x.s_o, w.causal, w.clip_c)
        runs.append((w, x, [_host(a, True) for a in (x.q, x.k, x.v)],
                     torch.empty(x.q.shape, dtype=torch.int8).pin_memory(), want))
    ws = torch.empty(ia.forward_host_workspace_size(2, 3, 150, 150, 64), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()

    def call_all():
        for w, x, (q, k, v), out, _ in runs:
            ia.forward_host(q, k, v, ia.Scales(x.s_q, x.s_k, x.s_v, x.s_o, per_head=True), w.causal, w.clip_c,
                            out=out, workspace=ws, stream=s)

    def check(what):
        for i, (_, _, _, out, want) in enumerate(runs):
            assert np.array_equal(out.numpy(), want), f"{what}: call {i} differs from the oracle"
            out.fill_(0x5A)

    with torch.cuda.stream(s):
        call_all()
        s.synchronize()
        check("warm-up")
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            call_all()
        for rep in range(2):
            g.replay()
            s.synchronize()
            check(f"replay {rep}")
        call_all()  # uncaptured again, after the capture, on the same workspace
        s.synchronize()
        check("after capture")
    del g
    assert ia.device_error() == ia.OK
