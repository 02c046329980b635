"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times (same plan, same kernels).  The single ViT-L step and block 0
of the 24-block stream at its last frame are compared on every output
element; the other checkpoints on sampled query rows that the oracle computes
one by one."""
import numpy as np
import pytest
import torch

from alloc_model import AllocModel
from gpu_util import (FrameBank, TOL_REL_L2, assert_close, gather_visible, make_cache,
                      max_pages_for, oracle_out, oracle_stream, rel_l2)
from streaming_video_transformer_b200.inputs import WORKLOADS, keyframe_decisions

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _rows(nq, n, seed):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(nq, size=n - 3, replace=False).tolist()) | {0, nq - 1, 128}
    return np.array(sorted(x for x in r if x < nq))


def test_vitl_step_full_size():
    """One 1375-token frame over ~99.8k visible tokens after 200 frames."""
    w = WORKLOADS["vitl_step"]
    prefill = w.frames - 1
    mp = max_pages_for(w, [w.frames])
    c = make_cache(w, mp)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(w.frames):
        q, k, v = bank.device(t)
        c.append_frame(0, k, v)
        c.evict_frames()
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq])
    info = c.plan_info()
    assert info["kv_tokens"][0] == st.num_visible_tokens() == 72 * 1369 + 6 * w.frames
    lse = torch.empty((w.Nq, w.H), dtype=torch.float32, device="cuda")
    out = c.run(0, q, lse=lse)
    out32 = c.run(0, q, force_fp32=True)
    # every query row and head: 1375 x 16 x 64 outputs
    ref, ref_lse = oracle_out(st, bank.oracle(prefill)[0])
    assert_close(out, ref, what="bf16")
    assert_close(out32, ref, fp32=True, what="fp32")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)
    # pool through the device table, bit for bit
    gk, gv = gather_visible(c, 0, 0)
    ok, ov = st.visible_kv()
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    # single-chunk plan gives the same result within tolerance
    c2 = make_cache(w, mp, max_splits=1)
    for t in range(w.frames):
        q, k, v = bank.device(t)
        c2.append_frame(0, k, v)
        c2.evict_frames()
    c2.build_visible_page_table()
    c2.plan([w.Nq])
    assert c2.plan_info()["splits"] == [1]
    assert info["splits"][0] > 1
    out1 = c2.run(0, q)
    assert rel_l2(out1.double().cpu().numpy(), out.double().cpu().numpy()) < TOL_REL_L2
    c.device_error()
    c2.device_error()


def test_vitl_stream24_blocks_0_and_23():
    """24 blocks, 1000 frames, 2-D RoPE; blocks 0 and 23 checked at chosen frames."""
    w = WORKLOADS["vitl_stream24"]
    checks = {1, 2, 8, 9, 72, 73, 74, 500, 1000}
    mp = max_pages_for(w, [w.frames])
    c = make_cache(w, mp)
    banks = {b: FrameBank(w, b, 0) for b in (0, 23)}
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    filler = [tuple(torch.randn((w.Nq, w.H, w.D), generator=g, device="cuda").to(torch.bfloat16)
                    for _ in range(3)) for _ in range(2)]
    sts = {b: oracle_stream(w) for b in (0, 23)}
    m = AllocModel(mp, w.P, w.ns, w.S, w.W)
    for t in range(w.frames):
        for b in range(w.blocks):
            src = banks[b].device(t) if b in banks else filler[t % 2]
            c.append_frame(b, src[1], src[2])
        c.evict_frames()
        m.append(0); m.evict(0)
        for b in banks:
            sts[b].append_frame(*banks[b].oracle(t)[1:])
        if t + 1 in checks:
            c.build_visible_page_table()
            c.plan([w.Nq])
            assert list(c.get_page_table()[1]) == m.table()[1]
            for b in banks:
                # block 0 at the last frame: every output element
                rows = (np.arange(w.Nq) if (b == 0 and t + 1 == w.frames)
                        else _rows(w.Nq, 24, t))
                out = c.run(b, banks[b].device(t)[0])
                ref, _ = oracle_out(sts[b], banks[b].oracle(t)[0], rows)
                assert_close(out[rows], ref, what=f"block {b} t={t + 1}")
    # RoPE'd keys in the pool: the oracle's fp32 rotation, bit for bit
    gk, gv = gather_visible(c, 23, 0)
    ok, ov = sts[23].visible_kv()
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    c.device_error()


def test_ragged4_batched_fp16_d128():
    """Four streams aged 10/70/300/2000 in one pool; one batched run."""
    w = WORKLOADS["ragged4"]
    ages = list(w.ages)
    mp = max_pages_for(w, ages, num_streams=4)
    c = make_cache(w, mp, num_streams=4)
    m = AllocModel(mp, w.P, w.ns, w.S, w.W, num_streams=4)
    banks = [FrameBank(w, 0, s) for s in range(4)]
    sts = [oracle_stream(w) for _ in range(4)]
    for s, age in enumerate(ages):
        for t in range(age):
            c.append_frame(0, *banks[s].device(t)[1:], stream=s)
            c.evict_frames(s)
            m.append(s); m.evict(s)
            sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq] * 4)
    dip, dix, dlp = c.read_device_page_table()
    mip, mix, mlp = m.table()
    assert list(dix) == mix and list(dip) == mip and list(dlp) == mlp
    assert [mip[i + 1] - mip[i] for i in range(4)] == [11, 37, 39, 52]
    assert list(dlp) == [60, 420, 232, 240]
    q = torch.cat([banks[s].device(ages[s] - 1)[0] for s in range(4)])
    out = c.run(0, q)
    assert out.dtype == torch.float16
    out32 = c.run(0, q, force_fp32=True)
    for s in range(4):
        rows = _rows(w.Nq, 24, s)
        ref, _ = oracle_out(sts[s], banks[s].oracle(ages[s] - 1)[0], rows)
        assert_close(out[s * w.Nq + rows], ref, what=f"stream {s}")
        assert_close(out32[s * w.Nq + rows], ref, fp32=True, what=f"fp32 stream {s}")
        gk, gv = gather_visible(c, 0, s)
        ok, ov = sts[s].visible_kv()
        assert np.array_equal(gk, ok) and np.array_equal(gv, ov)
    c.device_error()


@pytest.mark.parametrize("mode", ["bf16", "fp32_pool"])
def test_rollback10k_long_stream(mode):
    """10,000 offered frames, every 3rd deferred and rejected with p=0.3."""
    w = WORKLOADS["rollback10k"]
    if mode == "fp32_pool":
        from dataclasses import replace
        w = replace(w, dtype="fp32")
    dec = keyframe_decisions(w, w.frames)
    n_acc = sum(1 for d, r in dec if not r)
    mp = max_pages_for(w, [n_acc + 1])
    c = make_cache(w, mp)
    m = AllocModel(mp, w.P, w.ns, w.S, w.W)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    rejected_at = [t for t, (d, r) in enumerate(dec) if r]
    checks = {rejected_at[0], rejected_at[0] + 1, rejected_at[len(rejected_at) // 2],
              rejected_at[-1], rejected_at[-1] + 1, w.frames - 1}
    checked = 0
    for t, (deferred, rejected) in enumerate(dec):
        q, k, v = bank.device(t)
        c.set_defer_eviction(deferred)
        m.st[0].defer = deferred
        c.append_frame(0, k, v)
        c.evict_frames()
        m.append(0); m.evict(0)
        st.append_frame(*bank.oracle(t)[1:], deferred=deferred)
        if t in checks:
            c.build_visible_page_table()
            c.plan([w.Nq])
            assert list(c.get_page_table()[1]) == m.table()[1]
            rows = _rows(w.Nq, 16, t)
            ref, _ = oracle_out(st, bank.oracle(t)[0], rows)
            if mode == "bf16":
                assert_close(c.run(0, q)[rows], ref, what=f"t={t}")
            assert_close(c.run(0, q, force_fp32=True)[rows], ref, fp32=True, what=f"fp32 t={t}")
            checked += 1
        if deferred:
            if rejected:
                c.rollback_last_frame(); m.rollback(0); st.rollback_last_frame()
            else:
                c.execute_deferred_eviction(); m.accept(0); st.execute_deferred_eviction()
    assert checked == len(checks)
    s = c.get_cache_stats()
    assert s["frame_count"] == n_acc and s["special_tokens"] == 6 * n_acc
    assert s["scale_pages"] + s["live_pages"] == 72
    c.device_error()
