"""svt_frame_step, with and without CUDA-graph replay (GPU).

A whole frame step from one call: the appends of every block, eviction, the
visible table, the plan and the attention of every block.  With use_graph the
step's launches run as one CUDA graph, built for the first step of a launch
sequence and replayed with new kernel arguments afterwards.  Outputs must be
bit-identical to the separate calls, tables must match, and the results must
match the oracle."""
import numpy as np
import pytest
import torch

from gpu_util import (FrameBank, assert_close, gather_visible, make_cache, max_pages_for,
                      oracle_out, oracle_stream)
from streaming_video_transformer_b200.inputs import WORKLOADS, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _separate(c, w, ks, vs, qs):
    for b in range(w.blocks):
        c.append_frame(b, ks[b], vs[b])
    c.evict_frames()
    c.build_visible_page_table()
    c.plan([w.Nq])
    return [c.run(b, qs[b]) for b in range(w.blocks)]


def _out_like(w, qs, fp32=False):
    return [torch.empty(q.shape, dtype=torch.float32 if fp32 else q.dtype, device=q.device)
            for q in qs]


@pytest.mark.parametrize("case", ["tiny_stream", "two_blocks_rope", "fp32_pool"])
def test_frame_step_matches_separate_calls_and_oracle(case):
    if case == "tiny_stream":
        w = WORKLOADS["tiny_stream"]
    elif case == "two_blocks_rope":
        w = small_workload(P=16, ns=6, S=2, W=3, H=2, D=64, frames=10, R=10, blocks=2,
                           rope_grid=4)
    else:
        w = small_workload(P=36, ns=6, S=1, W=3, H=2, D=64, frames=8, R=8, dtype="fp32")
    mp = max_pages_for(w, [w.frames])
    caches = [make_cache(w, mp) for _ in range(3)]    # separate calls, step, step + graph
    banks = [FrameBank(w, b, 0, need_oracle=(b == 0)) for b in range(w.blocks)]
    st = oracle_stream(w)
    fp32 = w.dtype == "fp32"
    for t in range(w.frames):
        ks = [banks[b].device(t)[1] for b in range(w.blocks)]
        vs = [banks[b].device(t)[2] for b in range(w.blocks)]
        qs = [banks[b].device(t)[0] for b in range(w.blocks)]
        ref_outs = _separate(caches[0], w, ks, vs, qs)
        o1 = caches[1].frame_step(ks, vs, qs, _out_like(w, qs, fp32), use_graph=False)
        o2 = caches[2].frame_step(ks, vs, qs, _out_like(w, qs, fp32), use_graph=True)
        for b in range(w.blocks):
            assert torch.equal(o1[b], ref_outs[b]), f"t={t} block {b}"
            assert torch.equal(o2[b], ref_outs[b]), f"graph t={t} block {b}"
        tabs = [c.get_page_table() for c in caches]
        for tab in tabs[1:]:
            for a, bb in zip(tabs[0], tab):
                assert np.array_equal(a, bb)
        q64, k64, v64 = banks[0].oracle(t)
        st.append_frame(k64, v64)
        ref, _ = oracle_out(st, q64)
        assert_close(o2[0], ref, what=f"{case} t={t + 1}")
        gk, gv = gather_visible(caches[2], 0, 0)
        ok, ov = st.visible_kv()
        assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    builds, replays = caches[2].graph_counts()
    assert builds + replays == w.frames
    assert 1 <= builds <= 3 and replays >= w.frames - 3
    for c in caches:
        c.device_error()


def test_frame_step_graph_with_deferral_and_rollback():
    """Deferred frames attend through the graph step and are then accepted or
    rolled back on the host; every output equals the separate calls'."""
    w = small_workload(P=64, ns=6, S=2, W=3, H=2, D=64, frames=14, R=14, blocks=2)
    mp = max_pages_for(w, [w.frames])
    a, g = make_cache(w, mp), make_cache(w, mp)
    banks = [FrameBank(w, b, 0, need_oracle=False) for b in range(w.blocks)]
    rng = np.random.default_rng(7)
    for t in range(w.frames):
        deferred = t % 3 == 2
        ks = [banks[b].device(t)[1] for b in range(w.blocks)]
        vs = [banks[b].device(t)[2] for b in range(w.blocks)]
        qs = [banks[b].device(t)[0] for b in range(w.blocks)]
        for c in (a, g):
            c.set_defer_eviction(deferred)
        ref = _separate(a, w, ks, vs, qs)
        got = g.frame_step(ks, vs, qs, _out_like(w, qs), use_graph=True)
        for b in range(w.blocks):
            assert torch.equal(got[b], ref[b]), f"t={t} block {b}"
        if deferred:
            reject = rng.random() < 0.5
            for c in (a, g):
                (c.rollback_last_frame if reject else c.execute_deferred_eviction)()
        for x, y in zip(a.get_page_table(), g.get_page_table()):
            assert np.array_equal(x, y)
    a.device_error()
    g.device_error()


def test_frame_step_reports_errors_and_keeps_state():
    """A step on a stream whose last frame is still provisional is refused
    before anything changes; the next valid step runs normally."""
    from streaming_video_transformer_b200 import _lib
    from streaming_video_transformer_b200.cache import SvtError
    w = WORKLOADS["tiny_stream"]
    c = make_cache(w, max_pages_for(w, [4]))
    bank = FrameBank(w, 0, 0, need_oracle=False)
    q, k, v = bank.device(0)
    c.set_defer_eviction(True)
    c.frame_step([k], [v], [q], [torch.empty_like(q)])
    table = c.get_page_table()
    with pytest.raises(SvtError) as e:
        c.frame_step([k], [v], [q], [torch.empty_like(q)])
    assert e.value.code == _lib.SVT_ESTATE
    for x, y in zip(table, c.get_page_table()):
        assert np.array_equal(x, y)
    c.execute_deferred_eviction()
    c.set_defer_eviction(False)
    c.frame_step([k], [v], [q], [torch.empty_like(q)])
    c.device_error()


def test_frame_step_graph_at_full_size():
    """The 24-block ViT-L stream with 2-D RoPE: after the steady-state
    pre-fill, frame steps through svt_frame_step with graph replay give
    outputs bit-identical to the separate calls for every block."""
    from dataclasses import replace
    w = replace(WORKLOADS["vitl_stream24"], R=2)
    frames = w.S + w.W + 4
    mp = max_pages_for(w, [frames])
    a, g = make_cache(w, mp), make_cache(w, mp)
    banks = [FrameBank(w, b, 0, need_oracle=False) for b in range(w.blocks)]
    for t in range(w.S + w.W):
        for c in (a, g):
            for b in range(w.blocks):
                c.append_frame(b, *banks[b].device(t)[1:])
            c.evict_frames()
    for t in range(w.S + w.W, frames):
        ks = [banks[b].device(t)[1] for b in range(w.blocks)]
        vs = [banks[b].device(t)[2] for b in range(w.blocks)]
        qs = [banks[b].device(t)[0] for b in range(w.blocks)]
        ref = _separate(a, w, ks, vs, qs)
        got = g.frame_step(ks, vs, qs, _out_like(w, qs), use_graph=True)
        for b in range(w.blocks):
            assert torch.equal(got[b], ref[b]), f"t={t} block {b}"
        for x, y in zip(a.get_page_table(), g.get_page_table()):
            assert np.array_equal(x, y)
    # the one-launch append of all 24 blocks wrote the same pool bytes
    assert torch.equal(a.pool, g.pool)
    builds, replays = g.graph_counts()
    assert builds + replays == frames - w.S - w.W and builds <= 2
    a.device_error()
    g.device_error()


def test_frame_step_on_the_second_stream_of_a_shared_pool():
    """Two streams in one pool: stream 0 holds history, frame steps (graph
    replay) run on stream 1; outputs and tables equal the separate calls',
    and stream 0's part of the table is untouched."""
    w = small_workload(P=16, ns=6, S=2, W=3, H=2, D=64, frames=9, R=9, blocks=2)
    mp = max_pages_for(w, [w.frames, w.frames], num_streams=2)
    a, g = make_cache(w, mp, num_streams=2), make_cache(w, mp, num_streams=2)
    b0 = [FrameBank(w, b, 0, need_oracle=False) for b in range(w.blocks)]
    b1 = [FrameBank(w, b, 1, need_oracle=(b == 0)) for b in range(w.blocks)]
    for c in (a, g):
        for t in range(5):
            for b in range(w.blocks):
                c.append_frame(b, *b0[b].device(t)[1:], stream=0)
            c.evict_frames(0)
    st = oracle_stream(w)
    for t in range(w.frames):
        ks = [b1[b].device(t)[1] for b in range(w.blocks)]
        vs = [b1[b].device(t)[2] for b in range(w.blocks)]
        qs = [b1[b].device(t)[0] for b in range(w.blocks)]
        for b in range(w.blocks):
            a.append_frame(b, ks[b], vs[b], stream=1)
        a.evict_frames(1)
        a.build_visible_page_table()
        a.plan([0, w.Nq])
        ref = [a.run(b, qs[b]) for b in range(w.blocks)]
        got = g.frame_step(ks, vs, qs, _out_like(w, qs), stream=1, use_graph=True)
        for b in range(w.blocks):
            assert torch.equal(got[b], ref[b]), f"t={t} block {b}"
        for x, y in zip(a.get_page_table(), g.get_page_table()):
            assert np.array_equal(x, y)
        st.append_frame(*b1[0].oracle(t)[1:])
        o, _ = oracle_out(st, b1[0].oracle(t)[0])
        assert_close(got[0], o, what=f"stream 1 t={t + 1}")
    assert torch.equal(a.pool, g.pool)
    a.device_error()
    g.device_error()
