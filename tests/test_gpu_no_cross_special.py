"""GPU parity without cross-frame special retention
(kv_cache_cross_frame_special = False): a frame's special tokens are visible
exactly while its patch tokens are, and are stored after them in the frame's
own page.  Tables, pool bytes and outputs against the allocator model and the
oracle, from the tiny stream up to the ViT-L-sized step."""
import numpy as np
import pytest
import torch

import golden_io
from alloc_model import AllocModel
from gpu_util import (FrameBank, assert_close, gather_visible, make_cache, oracle_out,
                      oracle_stream_for)
from oracle import attend_lse
from streaming_video_transformer_b200.inputs import WORKLOADS, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _pages(w, streams=1):
    return streams * (w.S + w.W + 1)


def _frame(c, w, bank, t, stream=0, deferred=False):
    q, k, v = bank.device(t)
    c.set_defer_eviction(deferred, stream)
    for b in range(w.blocks):
        c.append_frame(b, k, v, stream=stream)
    c.evict_frames(stream)
    return q


def _check_step(c, w, st, m, q, q64, what):
    c.build_visible_page_table()
    c.plan([w.Nq])
    dip, dix, dlp = c.read_device_page_table()
    hip, hix, hlp = c.get_page_table()
    mip, mix, mlp = m.table()
    assert list(dip) == list(hip) == mip and list(dix) == list(hix) == mix, what
    assert list(dlp) == list(hlp) == mlp, what
    gk, gv = gather_visible(c, 0, 0)
    ok, ov = st.visible_kv()
    assert gk.shape[0] == st.num_visible_tokens()
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov), what
    ref, ref_lse = oracle_out(st, q64)
    lse = torch.empty((w.Nq, w.H), dtype=torch.float32, device="cuda")
    assert_close(c.run(0, q, lse=lse), ref, what=what)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)
    assert_close(c.run(0, q, force_fp32=True), ref, fp32=True, what="fp32 " + what)


CASES = [
    dict(P=16, ns=6, S=2, W=4, H=2, D=64, frames=12),                       # the tiny stream
    dict(P=122, ns=6, S=1, W=3, H=2, D=64, frames=7),                       # 128-token pages
    dict(P=250, ns=6, S=2, W=2, H=3, D=64, frames=6),                       # 2 tiles + tail
    dict(P=64, ns=6, S=0, W=3, H=2, D=128, frames=6, dtype="fp16"),         # no scale frames
    dict(P=100, ns=6, S=1, W=0, H=2, D=128, frames=4, rope_grid=10),        # empty window, RoPE
    dict(P=36, ns=6, S=2, W=2, H=2, D=64, frames=6, rope_grid=6, dtype="fp32"),
]


@pytest.mark.parametrize("cfg", CASES, ids=[str(i) for i in range(len(CASES))])
def test_stream_every_frame(cfg):
    w = small_workload(**cfg, R=cfg["frames"])
    c = make_cache(w, _pages(w), cross_frame_special=False)
    m = AllocModel(_pages(w), w.P, w.ns, w.S, w.W, cross_frame_special=False)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream_for(c, w)
    for t in range(w.frames):
        q = _frame(c, w, bank, t)
        m.append(0); m.evict(0)
        q64, k64, v64 = bank.oracle(t)
        st.append_frame(k64, v64)
        _check_step(c, w, st, m, q, q64, f"{cfg} t={t + 1}")
        s = c.get_cache_stats()
        assert s["special_tokens"] == w.ns * (s["scale_pages"] + s["live_pages"])
    c.device_error()


def test_hand_worked_example_without_retention():
    """The two-frame closed form without retention, embedded in D=64 as in the
    retained case (q scaled by 4 so that q.k/sqrt(64) = the example's q.k/2)."""
    cases, _ = golden_io.two_frame_cases(cross_frame_special=False)
    D = 64

    def pad(rows):
        x = torch.zeros((3, 1, D), dtype=torch.bfloat16)
        for i, r in enumerate(rows):
            x[i, 0, :4] = torch.tensor(r, dtype=torch.bfloat16)
        return x.cuda()

    q = pad([[8, 0, 0, 0], [0] * 4, [0] * 4])
    f0 = (pad([[1, 0, 0, 0], [0] * 4, [0] * 4]), pad([[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 1, 0]]))
    f1 = (pad([[0] * 4, [1, 0, 0, 0], [0] * 4]), pad([[0, 0, 0, 1], [1, 1, 0, 0], [0] * 4]))
    for S, W, t, row, expected in cases:
        w = small_workload(P=2, ns=1, S=S, W=W, H=1, D=D)
        c = make_cache(w, max_pages=S + W + 1, cross_frame_special=False)
        for k, v in (f0, f1)[:t]:
            c.append_frame(0, k, v)
            c.evict_frames()
        c.build_visible_page_table()
        c.plan([3])
        out = c.run(0, q).float().cpu().numpy()
        np.testing.assert_allclose(out[row, 0, :4], expected, atol=4e-3)
        out32 = c.run(0, q, force_fp32=True).cpu().numpy()
        np.testing.assert_allclose(out32[row, 0, :4], expected, atol=1e-6)


def test_deferred_frames_and_rollback():
    """Every third frame deferred, half of them rejected: the provisional
    frame's specials are visible with it and leave with a rollback; accepted
    frames evict the oldest window frame with its specials."""
    w = small_workload(P=40, ns=6, S=2, W=3, H=2, D=64, R=16, frames=16)
    c = make_cache(w, _pages(w), cross_frame_special=False)
    m = AllocModel(_pages(w), w.P, w.ns, w.S, w.W, cross_frame_special=False)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream_for(c, w)
    rng = np.random.default_rng(42)
    for t in range(w.frames):
        deferred = t % 3 == 2
        m.st[0].defer = deferred
        q = _frame(c, w, bank, t, deferred=deferred)
        m.append(0); m.evict(0)
        q64, k64, v64 = bank.oracle(t)
        st.append_frame(k64, v64, deferred=deferred)
        _check_step(c, w, st, m, q, q64, f"t={t + 1} deferred={deferred}")
        if deferred:
            if rng.random() < 0.5:
                c.rollback_last_frame(); m.rollback(0); st.rollback_last_frame()
            else:
                c.execute_deferred_eviction(); m.accept(0); st.execute_deferred_eviction()
    c.device_error()


def test_vitl_step_full_size_without_retention():
    """ViT-L-sized step (H16, D64, 1369 patches, S8, W64) at t = 120 frames:
    72 visible frames of 1375 tokens each (99,000 keys), sampled rows against
    the oracle, the pool bit for bit, and the table against the model."""
    w = WORKLOADS["vitl_step"]
    frames = 120
    c = make_cache(w, _pages(w), cross_frame_special=False)
    m = AllocModel(_pages(w), w.P, w.ns, w.S, w.W, cross_frame_special=False)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream_for(c, w)
    for t in range(frames):
        q = _frame(c, w, bank, t)
        m.append(0); m.evict(0)
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq])
    assert list(c.get_page_table()[1]) == m.table()[1]
    info = c.plan_info()
    assert info["kv_tokens"][0] == st.num_visible_tokens() == 72 * 1375
    assert info["kv_tiles"][0] == 72 * 11
    rows = np.array(sorted({0, 3, 5, 6, 127, 128, 640, 1279, 1280, 1374}))
    ref, _ = oracle_out(st, bank.oracle(frames - 1)[0], rows)
    assert_close(c.run(0, q)[rows], ref, what="bf16")
    assert_close(c.run(0, q, force_fp32=True)[rows], ref, fp32=True, what="fp32")
    gk, gv = gather_visible(c, 0, 0)
    ok, ov = st.visible_kv()
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    c.device_error()


@pytest.mark.parametrize("cfg", [
    dict(P=122, ns=6, S=1, W=3, H=2, D=64, frames=7),                       # 128-token pages
    dict(P=100, ns=6, S=1, W=2, H=2, D=128, frames=5, rope_grid=10),        # D = 128, RoPE
])
def test_dense_segment_without_retention(cfg):
    """A non-keyframe attends through a dense K/V segment on a pool whose
    pages hold a frame's patches and specials: the segment's tiles follow
    the pages' (page_size + num_special)-token tiles; nothing is stored."""
    w = small_workload(**cfg, R=cfg["frames"] + 1)
    c = make_cache(w, _pages(w), cross_frame_special=False)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream_for(c, w)
    for t in range(w.frames):
        _frame(c, w, bank, t)
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    table, stats = c.get_page_table(), c.get_cache_stats()
    pool0 = c.pool.clone()
    q, k, v = bank.device(w.frames)
    c.plan([w.Nq], extra_len=[w.Nq])
    assert c.plan_info()["kv_tokens"][0] == st.num_visible_tokens() + w.Nq
    out = c.run(0, q, k_extra=k, v_extra=v)
    out32 = c.run(0, q, k_extra=k, v_extra=v, force_fp32=True)
    q64, k64, v64 = bank.oracle(w.frames)
    kc, vc = st.visible_kv()
    ref, _ = attend_lse(q64, np.concatenate([kc, k64]), np.concatenate([vc, v64]))
    assert_close(out, ref, what="segment")
    assert_close(out32, ref, fp32=True, what="segment fp32")
    assert torch.equal(c.pool, pool0)
    for a, b in zip(table, c.get_page_table()):
        assert np.array_equal(a, b)
    assert c.get_cache_stats() == stats
    c.device_error()


def test_frame_step_graph_without_retention():
    """svt_frame_step with graph replay on a pool without retention (two
    blocks, the batched append writing each frame's specials after its
    patches): outputs, tables and pool bytes equal the separate calls'."""
    w = small_workload(P=40, ns=6, S=2, W=3, H=2, D=64, frames=10, R=10, blocks=2)
    a = make_cache(w, _pages(w), cross_frame_special=False)
    g = make_cache(w, _pages(w), cross_frame_special=False)
    banks = [FrameBank(w, b, 0, need_oracle=(b == 0)) for b in range(w.blocks)]
    st = oracle_stream_for(a, w)
    for t in range(w.frames):
        ks = [banks[b].device(t)[1] for b in range(w.blocks)]
        vs = [banks[b].device(t)[2] for b in range(w.blocks)]
        qs = [banks[b].device(t)[0] for b in range(w.blocks)]
        for b in range(w.blocks):
            a.append_frame(b, ks[b], vs[b])
        a.evict_frames()
        a.build_visible_page_table()
        a.plan([w.Nq])
        ref = [a.run(b, qs[b]) for b in range(w.blocks)]
        got = g.frame_step(ks, vs, qs, [torch.empty_like(q) for q in qs], use_graph=True)
        for b in range(w.blocks):
            assert torch.equal(got[b], ref[b]), f"t={t} block {b}"
        for x, y in zip(a.get_page_table(), g.get_page_table()):
            assert np.array_equal(x, y)
        st.append_frame(*banks[0].oracle(t)[1:])
        o, _ = oracle_out(st, banks[0].oracle(t)[0])
        assert_close(got[0], o, what=f"t={t + 1}")
    assert torch.equal(a.pool, g.pool)
    builds, replays = g.graph_counts()
    assert builds + replays == w.frames and replays >= w.frames - 3
    a.device_error()
    g.device_error()


def test_multi_frame_first_pass_without_retention():
    """Three frames appended, then all of their queries attend at once over
    the frames' patches and specials (no mask among them), with RoPE."""
    w = small_workload(P=36, ns=6, S=4, W=4, H=2, D=64, R=8, rope_grid=6)
    F = 3
    c = make_cache(w, _pages(w), cross_frame_special=False, max_qo_len=F * w.Nq)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream_for(c, w)
    for t in range(F):
        _frame(c, w, bank, t)
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([F * w.Nq])
    assert c.plan_info()["kv_tokens"][0] == st.num_visible_tokens() == F * w.Nq
    q = torch.cat([bank.device(t)[0] for t in range(F)])
    q64 = np.concatenate([bank.oracle(t)[0] for t in range(F)])
    ref, _ = oracle_out(st, q64)
    assert_close(c.run(0, q), ref, what="first pass")
    assert_close(c.run(0, q, force_fp32=True), ref, fp32=True, what="first pass fp32")
    c.device_error()


def test_two_streams_batched_without_retention():
    """Two streams of different ages in one pool without retention, one
    batched run: each stream's rows against its own oracle stream."""
    w = small_workload(P=60, ns=6, S=2, W=3, H=2, D=64, R=12)
    ages = [4, 11]
    c = make_cache(w, 2 * _pages(w), num_streams=2, cross_frame_special=False)
    banks = [FrameBank(w, 0, s) for s in range(2)]
    sts = [oracle_stream_for(c, w) for _ in range(2)]
    for s, age in enumerate(ages):
        for t in range(age):
            _frame(c, w, banks[s], t, stream=s)
            sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq, w.Nq])
    q = torch.cat([banks[s].device(ages[s] - 1)[0] for s in range(2)])
    out = c.run(0, q)
    out32 = c.run(0, q, force_fp32=True)
    for s in range(2):
        ref, _ = oracle_out(sts[s], banks[s].oracle(ages[s] - 1)[0])
        assert_close(out[s * w.Nq:(s + 1) * w.Nq], ref, what=f"stream {s}")
        assert_close(out32[s * w.Nq:(s + 1) * w.Nq], ref, fp32=True, what=f"fp32 stream {s}")
    c.device_error()
