"""svt_attention_noalloc against svt_run (GPU).

The allocation-free entry point serves callers that cannot allocate device
memory (an allocator that is locked or forbidden, a framework that owns all
device buffers, a fixed memory budget): it keeps its split-KV scratch in a
fixed array inside the library.  Here it is called twice in a row through the
C ABI and each result is compared with svt_run on the same cache, within the
tolerance the parity tests use.  The test allocates its own inputs; the entry
point itself allocates nothing.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from gpu_util import FrameBank, TOL_MAX_ABS, TOL_REL_L2, make_cache, max_pages_for, rel_l2
from streaming_video_transformer_b200 import _lib
from streaming_video_transformer_b200.cache import SvtError, attention_noalloc
from streaming_video_transformer_b200.inputs import WORKLOADS, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _filled(w, ages):
    c = make_cache(w, max_pages_for(w, ages, num_streams=len(ages)), num_streams=len(ages))
    banks = [FrameBank(w, 0, s, need_oracle=False) for s in range(len(ages))]
    for s, age in enumerate(ages):
        for t in range(age):
            c.append_frame(0, *banks[s].device(t)[1:], stream=s)
            c.evict_frames(s)
    c.build_visible_page_table()
    c.plan([w.Nq] * len(ages))
    q = torch.cat([banks[s].device(ages[s] - 1)[0] for s in range(len(ages))])
    return c, q


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.all(np.isfinite(a))
    assert float(np.max(np.abs(a - b))) <= TOL_MAX_ABS
    assert rel_l2(a, b) <= TOL_REL_L2


@pytest.mark.parametrize("case", ["vitl_bf16", "ragged_fp16_d128"])
def test_noalloc_matches_run_twice(case):
    if case == "vitl_bf16":
        w, ages = WORKLOADS["vitl_step"], [90]
    else:
        w, ages = small_workload(H=4, D=128, P=784, ns=6, S=4, W=8, dtype="fp16", R=8), [5, 30]
    c, q = _filled(w, ages)
    ref_lse = torch.empty((q.shape[0], w.H), dtype=torch.float32, device="cuda")
    ref = c.run(0, q, lse=ref_lse)
    ip, ix, lp = c.get_page_table()
    indices = torch.from_numpy(ix).to("cuda")
    pool_block = c.pool[0]
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((q.shape[0], w.H), float("nan"), dtype=torch.float32, device="cuda")
        attention_noalloc(q, out, pool_block, indices, ip, lp, [w.Nq] * len(ages),
                          c.max_pages, w.P, lse=lse)
        torch.cuda.synchronize()
        _close(out, ref)
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=2e-2)


def test_noalloc_rejects_oversized_split_request():
    w = WORKLOADS["vitl_step"]
    c, q = _filled(w, [80])
    ip, ix, lp = c.get_page_table()
    indices = torch.from_numpy(ix).to("cuda")
    out = torch.empty_like(q)
    with pytest.raises(SvtError) as e:
        attention_noalloc(q, out, c.pool[0], indices, ip, lp, [w.Nq], c.max_pages, w.P,
                          num_splits=64)
    assert e.value.code == _lib.SVT_EINVAL
    assert "scratch" in str(e.value)
