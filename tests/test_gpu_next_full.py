"""GPU parity of the scheme's further uses at the ViT-L stream's full sizes,
in the configuration the benchmark measures them in (GPU).

- Multi-frame first pass: the 8 scale frames of the 2-D RoPE stream appended,
  then all 8 x 1375 queries attend over all 8 frames at once (no mask among
  them): every output element against the oracle.
- Skip-append: at the stream's steady state a non-keyframe attends over the
  cache plus its own K/V given as a dense segment; sampled rows against the
  oracle (the cache's visible K/V followed by the frame's rows), with the
  pool, page table and statistics unchanged afterwards."""
from dataclasses import replace

import numpy as np
import pytest
import torch

from gpu_util import (FrameBank, assert_close, make_cache, max_pages_for, oracle_out,
                      oracle_stream)
from oracle import attend_lse
from streaming_video_transformer_b200.inputs import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _rows(nq, n, seed):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(nq, size=n - 4, replace=False).tolist()) | {0, 5, 6, nq - 1}
    return np.array(sorted(r))


def test_first_pass_8_frames_full_size():
    w = replace(WORKLOADS["vitl_stream24"], blocks=1, R=8)
    F = w.S
    c = make_cache(w, max_pages_for(w, [F]), max_qo_len=F * w.Nq)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(F):
        c.append_frame(0, *bank.device(t)[1:])
        c.evict_frames()
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([F * w.Nq])
    info = c.plan_info()
    assert info["kv_tokens"][0] == st.num_visible_tokens() == F * w.Nq
    q = torch.cat([bank.device(t)[0] for t in range(F)])
    q64 = np.concatenate([bank.oracle(t)[0] for t in range(F)])
    lse = torch.empty((F * w.Nq, w.H), dtype=torch.float32, device="cuda")
    out = c.run(0, q, lse=lse)
    ref, ref_lse = oracle_out(st, q64)          # 11,000 rows x 16 heads
    assert_close(out, ref, what="first pass, every element")
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=2e-2)
    rows = _rows(F * w.Nq, 48, 11)
    out32 = c.run(0, q, force_fp32=True)
    assert_close(out32[rows], ref[rows], fp32=True, what="first pass fp32")
    c.device_error()


def test_skip_append_dense_segment_full_size():
    w = replace(WORKLOADS["vitl_stream24"], blocks=1, R=4)
    pre = w.S + w.W + 8                          # steady state: 72 patch pages visible
    c = make_cache(w, max_pages_for(w, [pre + 1]), max_qo_len=w.Nq)
    bank = FrameBank(w, 0, 0)
    st = oracle_stream(w)
    for t in range(pre):
        c.append_frame(0, *bank.device(t)[1:])
        c.evict_frames()
        st.append_frame(*bank.oracle(t)[1:])
    c.build_visible_page_table()
    table, stats = c.get_page_table(), c.get_cache_stats()
    pool0 = c.pool.clone()
    q, k, v = bank.device(pre)
    c.plan([w.Nq], extra_len=[w.Nq])
    info = c.plan_info()
    assert info["kv_tokens"][0] == st.num_visible_tokens() + w.Nq
    assert info["splits"][0] > 1                 # the split-KV path, as the benchmark runs it
    out = c.run(0, q, k_extra=k, v_extra=v)
    out32 = c.run(0, q, k_extra=k, v_extra=v, force_fp32=True)
    q64, k64, v64 = bank.oracle(pre)
    kc, vc = st.visible_kv()
    rows = _rows(w.Nq, 32, 12)
    ref, _ = attend_lse(q64[rows], np.concatenate([kc, k64]), np.concatenate([vc, v64]))
    assert_close(out[rows], ref, what="dense segment")
    assert_close(out32[rows], ref, fp32=True, what="dense segment fp32")
    assert torch.equal(c.pool, pool0)
    for a, b in zip(table, c.get_page_table()):
        assert np.array_equal(a, b)
    assert c.get_cache_stats() == stats
    c.device_error()
