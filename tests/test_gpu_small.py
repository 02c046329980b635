"""GPU parity at small sizes: the tiny stream, the hand-worked example,
edge cases, and the invariants (page-id independence, rollback)."""
import numpy as np
import pytest
import torch

import golden_io
from alloc_model import AllocModel
from gpu_util import (FrameBank, assert_close, gather_visible, make_cache, max_pages_for,
                      oracle_out, oracle_stream)
from oracle import attend_lse
from streaming_video_transformer_b200 import _lib
from streaming_video_transformer_b200.inputs import WORKLOADS, frame_qkv, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _step(cache, w, bank, t, blocks=(0,), stream=0, deferred=False):
    q, k, v = bank.device(t)
    if deferred:
        cache.set_defer_eviction(True, stream)
    for b in range(w.blocks):
        cache.append_frame(b, k, v, stream=stream)
    cache.evict_frames(stream)
    cache.build_visible_page_table()
    cache.plan([w.Nq])
    return q


def test_tiny_stream_every_frame():
    """12 frames, one at a time: table, pool bytes and outputs every frame."""
    w = WORKLOADS["tiny_stream"]
    mp = max_pages_for(w, [w.frames])
    c = make_cache(w, mp)
    m = AllocModel(mp, w.P, w.ns, w.S, w.W)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    counts = [int(x) for x in golden_io.visible_counts()["tiny"][1]]
    for t in range(w.frames):
        q = _step(c, w, bank, t)
        m.append(0); m.evict(0)
        q64, k64, v64 = bank.oracle(t)
        st.append_frame(k64, v64)
        # page tables: device == host == model
        dip, dix, dlp = c.read_device_page_table()
        hip, hix, hlp = c.get_page_table()
        mip, mix, mlp = m.table()
        assert list(dip) == list(hip) == mip and list(dix) == list(hix) == mix
        assert list(dlp) == list(hlp) == mlp
        # pool through the table == oracle visible K/V, bit for bit
        gk, gv = gather_visible(c, 0, 0)
        ok, ov = st.visible_kv()
        assert gk.shape[0] == counts[t]
        assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
        ref, ref_lse = oracle_out(st, q64)
        lse = torch.empty((w.Nq, w.H), dtype=torch.float32, device="cuda")
        out = c.run(0, q, lse=lse)
        assert out.dtype == torch.bfloat16
        assert_close(out, ref, what=f"t={t + 1}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)
        out32 = c.run(0, q, force_fp32=True, lse=lse)
        assert out32.dtype == torch.float32
        assert_close(out32, ref, fp32=True, what=f"fp32 t={t + 1}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=1e-5)
    c.device_error()


def test_hand_worked_example_on_gpu():
    """The two-frame closed form, embedded in D=64 (zero features; q scaled
    by 4 so that q.k/sqrt(64) equals the example's q.k/sqrt(4))."""
    cases, _ = golden_io.two_frame_cases()
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
        c = make_cache(small_workload(P=2, ns=1, S=S, W=W, H=1, D=D), max_pages=12)
        for k, v in (f0, f1)[:t]:
            c.append_frame(0, k, v)
            c.evict_frames()
        c.build_visible_page_table()
        c.plan([3])
        out = c.run(0, q).float().cpu().numpy()
        np.testing.assert_allclose(out[row, 0, :4], expected, atol=4e-3)
        np.testing.assert_array_equal(out[row, 0, 4:], 0)
        out32 = c.run(0, q, force_fp32=True).cpu().numpy()
        np.testing.assert_allclose(out32[row, 0, :4], expected, atol=1e-6)


EDGE = [
    dict(P=16, ns=6, S=0, W=3, H=2, D=64, frames=7),              # no scale frames
    dict(P=16, ns=6, S=2, W=0, H=2, D=64, frames=5),              # empty window
    dict(P=8, ns=8, S=1, W=2, H=1, D=64, frames=6),               # last page always full
    dict(P=200, ns=6, S=2, W=3, H=3, D=64, frames=6),             # page > 128 tokens: 2 tiles
    dict(P=300, ns=6, S=1, W=2, H=2, D=128, frames=5, dtype="fp16"),
    dict(P=16, ns=0, S=2, W=2, H=2, D=64, frames=5),              # no special tokens
    dict(P=130, ns=6, S=3, W=4, H=4, D=64, frames=9),             # Nq 136: ragged q tile
    # D = 128 runs 64-token KV tiles: pages of one tile, of a tile and a
    # 36-row tail (with 2-D RoPE on a 10x10 grid), and of a quarter tile.
    dict(P=64, ns=6, S=2, W=2, H=2, D=128, frames=5),
    dict(P=100, ns=6, S=1, W=3, H=2, D=128, frames=6, rope_grid=10),
    dict(P=16, ns=6, S=2, W=3, H=2, D=128, frames=7, dtype="fp16"),
    # 2-D RoPE at D = 64 in fp16 (a 6x6 grid), and on an fp32 pool, where the
    # rotated keys are stored without a further rounding.
    dict(P=36, ns=6, S=1, W=2, H=2, D=64, frames=5, rope_grid=6, dtype="fp16"),
    dict(P=16, ns=6, S=1, W=2, H=2, D=64, frames=4, rope_grid=4, dtype="fp32"),
]


@pytest.mark.parametrize("cfg", EDGE, ids=[str(i) for i in range(len(EDGE))])
def test_edge_shapes(cfg):
    w = small_workload(**cfg, R=cfg["frames"])
    c = make_cache(w, max_pages_for(w, [w.frames]))
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(w.frames):
        q = _step(c, w, bank, t)
        q64, k64, v64 = bank.oracle(t)
        st.append_frame(k64, v64)
        ref, _ = oracle_out(st, q64)
        assert_close(c.run(0, q), ref, what=f"{cfg} t={t + 1}")
        assert_close(c.run(0, q, force_fp32=True), ref, fp32=True, what=f"fp32 {cfg} t={t + 1}")
        # pool through the device table == oracle visible K/V, bit for bit
        # (with RoPE: keys rotated by the same fp32 formula on both sides)
        gk, gv = gather_visible(c, 0, 0)
        ok, ov = st.visible_kv()
        assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    c.device_error()


def test_page_ids_do_not_change_outputs():
    w = small_workload(P=64, ns=6, S=2, W=3, H=2, D=64, frames=9, R=9)
    mp = max_pages_for(w, [w.frames])
    outs = []
    for perm in (False, True):
        c = make_cache(w, mp)
        if perm:
            rng = np.random.default_rng(3)
            c.set_free_lists(rng.permutation(c.patch_pages),
                             c.patch_pages + rng.permutation(mp - c.patch_pages))
        bank = FrameBank(w, 0, 0, need_oracle=False)
        for t in range(w.frames):
            q = _step(c, w, bank, t)
        outs.append((c.run(0, q).cpu(), c.run(0, q, force_fp32=True).cpu(), c.get_page_table()[1]))
    assert not np.array_equal(outs[0][2], outs[1][2])           # different physical pages
    assert torch.equal(outs[0][0], outs[1][0])                   # bit-identical outputs
    assert torch.equal(outs[0][1], outs[1][1])


def test_rollback_restores_outputs_bit_exactly():
    w = small_workload(P=64, ns=6, S=2, W=3, H=2, D=64, frames=12, R=12, blocks=2)
    c = make_cache(w, max_pages_for(w, [w.frames]))
    bank = FrameBank(w, 0, 0, need_oracle=False)
    for t in range(7):
        q = _step(c, w, bank, t)
    before = [c.run(b, q).cpu() for b in range(2)]
    table = c.get_page_table()
    q2 = _step(c, w, bank, 7, deferred=True)
    during = c.run(0, q2).cpu()
    c.rollback_last_frame()
    c.set_defer_eviction(False)
    c.build_visible_page_table()
    c.plan([w.Nq])
    after = [c.run(b, q).cpu() for b in range(2)]
    for a, b in zip(before, after):
        assert torch.equal(a, b)
    for a, b in zip(table, c.get_page_table()):
        assert np.array_equal(a, b)
    assert during.shape == before[0].shape


def test_multi_stream_with_idle_stream():
    """Three streams in one pool, the middle one has no query this step."""
    w = small_workload(P=32, ns=6, S=1, W=2, H=2, D=64, R=8)
    ages = [3, 5, 8]
    c = make_cache(w, max_pages_for(w, ages, num_streams=3), num_streams=3)
    banks = [FrameBank(w, 0, s) for s in range(3)]
    sts = [oracle_stream(w) for _ in range(3)]
    for s, age in enumerate(ages):
        for t in range(age):
            q, k, v = banks[s].device(t)
            c.append_frame(0, k, v, stream=s)
            c.evict_frames(s)
            sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq, 0, w.Nq])
    qa = banks[0].device(ages[0] - 1)[0]
    qc = banks[2].device(ages[2] - 1)[0]
    out = c.run(0, torch.cat([qa, qc]))
    for s, rows in ((0, slice(0, w.Nq)), (2, slice(w.Nq, 2 * w.Nq))):
        ref, _ = oracle_out(sts[s], banks[s].oracle(ages[s] - 1)[0])
        assert_close(out[rows], ref, what=f"stream {s}")


def test_skip_append_non_keyframe():
    """A frame that attends without being stored (the upstream skip-append
    path for non-keyframes): deferred append, attention, rollback.  Its
    queries see the cache plus its own tokens; afterwards the cache is as
    before, bit for bit."""
    w = small_workload(P=48, ns=6, S=2, W=3, H=2, D=64, R=16, blocks=2)
    c = make_cache(w, max_pages_for(w, [12]))
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(7):
        q = _step(c, w, bank, t)
        st.append_frame(*bank.oracle(t)[1:])
    table, stats = c.get_page_table(), c.get_cache_stats()
    gk0, gv0 = gather_visible(c, 0, 0)
    # skip-append frame 7
    q = _step(c, w, bank, 7, deferred=True)
    st.append_frame(*bank.oracle(7)[1:], deferred=True)
    ref, _ = oracle_out(st, bank.oracle(7)[0])
    assert_close(c.run(0, q), ref, what="skip-append frame")
    c.rollback_last_frame()
    c.set_defer_eviction(False)
    st.rollback_last_frame()
    for a, b in zip(table, c.get_page_table()):
        assert np.array_equal(a, b)
    assert c.get_cache_stats() == stats
    c.build_visible_page_table()
    gk1, gv1 = gather_visible(c, 0, 0)
    assert np.array_equal(gk0, gk1) and np.array_equal(gv0, gv1)
    # the next stored frame sees exactly the cache it would have seen
    q = _step(c, w, bank, 8)
    st.append_frame(*bank.oracle(8)[1:])
    ref, _ = oracle_out(st, bank.oracle(8)[0])
    assert_close(c.run(0, q), ref, what="frame after skip-append")


def test_multi_frame_first_pass_with_rope():
    """First pass over a clip: several frames appended, then all of their
    queries attend at once (no causal mask among them)."""
    w = small_workload(P=16, ns=6, S=4, W=4, H=2, D=64, R=8, rope_grid=4)
    F = 3
    c = make_cache(w, max_pages_for(w, [F]), max_qo_len=F * w.Nq)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(F):
        c.append_frame(0, *bank.device(t)[1:])
        c.evict_frames()
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([F * w.Nq])
    q = torch.cat([bank.device(t)[0] for t in range(F)])
    q64 = np.concatenate([bank.oracle(t)[0] for t in range(F)])
    ref, _ = oracle_out(st, q64)
    assert_close(c.run(0, q), ref, what="first pass")
    assert_close(c.run(0, q, force_fp32=True), ref, fp32=True, what="first pass fp32")


def test_bounded_wait_gives_up_and_context_stays_usable():
    """Failure detection without a fault: a kernel waits on an mbarrier that
    nothing arrives on; the bounded wait gives up and reports, and the GPU
    keeps working."""
    import time
    from streaming_video_transformer_b200 import _lib
    from streaming_video_transformer_b200.cache import SvtError, selftest_wait_limit
    t0 = time.perf_counter()
    with pytest.raises(SvtError) as e:
        selftest_wait_limit(20000)                 # 20 ms
    assert e.value.code == _lib.SVT_EDEVICE
    assert time.perf_counter() - t0 < 5.0
    w = WORKLOADS["tiny_stream"]
    c = make_cache(w, max_pages_for(w, [3]))
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(3):
        q = _step(c, w, bank, t)
        st.append_frame(*bank.oracle(t)[1:])
    ref, _ = oracle_out(st, bank.oracle(2)[0])
    assert_close(c.run(0, q), ref, what="after the self-test")
    c.device_error()


@pytest.mark.parametrize("splits", [1, 16])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("jump", [3.0, 60.0, 150.0, -150.0])
def test_row_max_jumps_in_later_tiles(dtype, jump, splits):
    """Keys whose scores sit `jump` log2 units above (or below) the rest
    appear in a late patch page and among the last special tokens (the
    partial last page), so that the running maximum taken from the earlier
    tiles is exceeded mid-row: by a little, by enough that the speculative
    exponentials exceed 2^8, and by enough that they overflow to +inf.
    With one KV chunk per row both jumps land in late tiles of one CTA (the
    last tile for the special key); with the planner's splits they may open
    a chunk."""
    w = small_workload(P=256, ns=6, S=1, W=3, H=2, D=64, frames=5, R=5, dtype=dtype)
    tdt = w.torch_dtype
    g = torch.Generator().manual_seed(5150)
    u = torch.zeros(w.D)
    u[7] = 1.0
    beta = 4.0                                     # shared q component along u
    alpha = jump * np.sqrt(w.D) / (np.log2(np.e) * beta)
    frames = []
    for t in range(w.frames):
        k = torch.randn((w.Nq, w.H, w.D), generator=g) / np.sqrt(w.D)
        v = torch.randn((w.Nq, w.H, w.D), generator=g)
        if t == w.frames - 2:
            k[w.ns + 100] = alpha * u              # a patch key of a late window page
        if t == w.frames - 1:
            k[2] = alpha * u                       # a special key on the last page
        frames.append((k.to(tdt), v.to(tdt)))
    q = (torch.randn((w.Nq, w.H, w.D), generator=g) / np.sqrt(w.D) + beta * u).to(tdt)
    c = make_cache(w, max_pages_for(w, [w.frames]), max_splits=splits)
    st = oracle_stream(w)
    for k, v in frames:
        c.append_frame(0, k.cuda(), v.cuda())
        c.evict_frames()
        st.append_frame(k.double().numpy(), v.double().numpy())
    c.build_visible_page_table()
    c.plan([w.Nq])
    if splits == 1:
        info = c.plan_info()
        assert info["splits"] == [1] and info["kv_tiles"][0] >= 9
    ref, lse_ref = oracle_out(st, q.double().numpy())
    lse = torch.empty((w.Nq, w.H), dtype=torch.float32, device="cuda")
    out = c.run(0, q.cuda(), lse=lse)
    assert_close(out, ref, what=f"{dtype} jump {jump}")
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-3, atol=2e-2)
    assert_close(c.run(0, q.cuda(), force_fp32=True), ref, fp32=True, what=f"fp32 jump {jump}")
    c.device_error()


SEGMENT = [
    dict(P=48, ns=6, S=2, W=3, H=2, D=64),                         # bf16
    dict(P=36, ns=6, S=1, W=2, H=2, D=64, rope_grid=6),            # 2-D RoPE on the segment's K
    dict(P=100, ns=6, S=1, W=3, H=2, D=128, dtype="fp16"),         # 64-token tiles, ragged tail
]


@pytest.mark.parametrize("cfg", SEGMENT, ids=[str(i) for i in range(len(SEGMENT))])
def test_skip_append_with_dense_segment(cfg):
    """A non-keyframe attends to the cache plus its own K/V given as a dense
    segment: nothing is written to the pool and the allocator is untouched.
    Stream 0 attends with its frame as a segment, stream 1 (in the same run)
    with its cache only."""
    w = small_workload(**cfg, R=16)
    c = make_cache(w, max_pages_for(w, [12, 12], num_streams=2), num_streams=2)
    banks = [FrameBank(w, 0, s) for s in range(2)]
    sts = [oracle_stream(w) for _ in range(2)]
    for s in range(2):
        for t in range(7):
            c.append_frame(0, *banks[s].device(t)[1:], stream=s)
            c.evict_frames(s)
            sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    table, stats = c.get_page_table(), c.get_cache_stats()
    pool0 = c.pool.clone()
    q7, k7, v7 = banks[0].device(7)
    q1 = banks[1].device(6)[0]
    c.plan([w.Nq, w.Nq], extra_len=[w.Nq, 0])
    info = c.plan_info()
    assert info["kv_tokens"][0] == sts[0].num_visible_tokens() + w.Nq
    q = torch.cat([q7, q1])
    out = c.run(0, q, k_extra=k7, v_extra=v7)
    out32 = c.run(0, q, k_extra=k7, v_extra=v7, force_fp32=True)
    q64, k64, v64 = banks[0].oracle(7)
    kc, vc = sts[0].visible_kv()
    ref0, _ = attend_lse(q64, np.concatenate([kc, k64]), np.concatenate([vc, v64]))
    ref1, _ = oracle_out(sts[1], banks[1].oracle(6)[0])
    assert_close(out[:w.Nq], ref0, what="segment stream")
    assert_close(out32[:w.Nq], ref0, fp32=True, what="segment stream fp32")
    assert_close(out[w.Nq:], ref1, what="plain stream")
    assert_close(out32[w.Nq:], ref1, fp32=True, what="plain stream fp32")
    # nothing stored, nothing allocated
    assert torch.equal(c.pool, pool0)
    for a, b in zip(table, c.get_page_table()):
        assert np.array_equal(a, b)
    assert c.get_cache_stats() == stats
    # the deferred append / attend / rollback route gives the same attention
    c.set_defer_eviction(True, 0)
    c.append_frame(0, k7, v7, stream=0)
    c.evict_frames(0)
    c.build_visible_page_table()
    c.plan([w.Nq, 0])
    via_pool = c.run(0, q7)
    assert_close(via_pool, out[:w.Nq].double().cpu().numpy(), what="segment vs deferred append")
    c.rollback_last_frame(0)
    c.set_defer_eviction(False, 0)
    # the next stored frame sees exactly the cache it would have seen
    c.append_frame(0, *banks[0].device(8)[1:], stream=0)
    c.evict_frames(0)
    sts[0].append_frame(*banks[0].oracle(8)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq, 0])
    ref, _ = oracle_out(sts[0], banks[0].oracle(8)[0])
    assert_close(c.run(0, banks[0].device(8)[0]), ref, what="frame after the segment step")
    c.device_error()


def test_dense_segment_on_a_stream_with_no_stored_frames():
    """The first frame of a stream attended as a non-keyframe: no pages are
    visible and every KV tile comes from the dense segment (bf16 and fp32
    paths, D = 64 and D = 128); the table stays empty."""
    for D, P in ((64, 200), (128, 100)):
        w = small_workload(P=P, ns=6, S=2, W=3, H=2, D=D, R=2)
        c = make_cache(w, max_pages_for(w, [2]))
        c.build_visible_page_table()
        q, k, v = FrameBank(w, 0, 0).device(0)
        q64, k64, v64 = FrameBank(w, 0, 0).oracle(0)
        c.plan([w.Nq], extra_len=[w.Nq])
        info = c.plan_info()
        assert info["kv_tokens"][0] == w.Nq
        ref, _ = attend_lse(q64, k64, v64)
        assert_close(c.run(0, q, k_extra=k, v_extra=v), ref, what=f"D={D}")
        assert_close(c.run(0, q, k_extra=k, v_extra=v, force_fp32=True), ref, fp32=True,
                     what=f"fp32 D={D}")
        ip, ix, lp = c.get_page_table()
        assert list(ip) == [0, 0] and len(ix) == 0
        c.device_error()


def test_batch_of_the_maximum_number_of_streams():
    """SVT_MAX_STREAMS (32) streams of different ages in one pool and one
    batched run; sampled streams against the oracle."""
    w = small_workload(P=16, ns=6, S=1, W=2, H=2, D=64, R=6)
    n = _lib.MAX_STREAMS
    ages = [1 + (s % 6) for s in range(n)]
    c = make_cache(w, max_pages_for(w, ages, num_streams=n), num_streams=n)
    banks = [FrameBank(w, 0, s, need_oracle=(s % 7 == 0)) for s in range(n)]
    sts = {s: oracle_stream(w) for s in range(0, n, 7)}
    for s, age in enumerate(ages):
        for t in range(age):
            c.append_frame(0, *banks[s].device(t)[1:], stream=s)
            c.evict_frames(s)
            if s in sts:
                sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq] * n)
    q = torch.cat([banks[s].device(ages[s] - 1)[0] for s in range(n)])
    out = c.run(0, q)
    for s, st in sts.items():
        ref, _ = oracle_out(st, banks[s].oracle(ages[s] - 1)[0])
        assert_close(out[s * w.Nq:(s + 1) * w.Nq], ref, what=f"stream {s}")
    c.device_error()
