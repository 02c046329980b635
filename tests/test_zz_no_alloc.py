"""svt_attention_noalloc against svt_run and against the oracle (GPU).

The allocation-free entry point serves callers that cannot allocate device
memory (an allocator that is locked or forbidden, a framework that owns all
device buffers, a fixed memory budget): it keeps its split-KV scratch in a
fixed array inside the library.  Here it is called twice in a row through the
C ABI and each result is compared with svt_run on the same cache, within the
tolerance the parity tests use, and with the CPU oracle.  The branches in which
it differs from svt_run are covered: the automatic split choice, an explicit
split count (1 = direct write, no merge), with and without an LSE buffer, and
a batch whose streams have very different KV lengths.  Its device error word
is read back through svt_noalloc_device_error.  The test allocates its own
inputs; the entry point itself allocates nothing.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from gpu_util import (FrameBank, TOL_MAX_ABS, TOL_REL_L2, assert_close, make_cache,
                      max_pages_for, oracle_out, oracle_stream, rel_l2)
from streaming_video_transformer_b200 import _lib
from streaming_video_transformer_b200.cache import (SvtError, attention_noalloc,
                                                     noalloc_device_error)
from streaming_video_transformer_b200.inputs import WORKLOADS, small_workload

pytestmark = pytest.mark.gpu

SCRATCH_FLOATS = (32 << 20) // 4


@pytest.fixture(scope="module", autouse=True)
def _build():
    from streaming_video_transformer_b200.build import build
    build()


def _filled(w, ages, oracle=False):
    c = make_cache(w, max_pages_for(w, ages, num_streams=len(ages)), num_streams=len(ages))
    banks = [FrameBank(w, 0, s, need_oracle=oracle) for s in range(len(ages))]
    sts = [oracle_stream(w) for _ in ages] if oracle else None
    for s, age in enumerate(ages):
        for t in range(age):
            c.append_frame(0, *banks[s].device(t)[1:], stream=s)
            c.evict_frames(s)
            if oracle:
                sts[s].append_frame(*banks[s].oracle(t)[1:])
    c.build_visible_page_table()
    c.plan([w.Nq] * len(ages))
    q = torch.cat([banks[s].device(ages[s] - 1)[0] for s in range(len(ages))])
    q64 = (np.concatenate([banks[s].oracle(ages[s] - 1)[0] for s in range(len(ages))])
           if oracle else None)
    return c, q, sts, q64


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    assert np.all(np.isfinite(a))
    assert float(np.max(np.abs(a - b))) <= TOL_MAX_ABS
    assert rel_l2(a, b) <= TOL_REL_L2


def _call(c, q, w, n_streams, lse=None, num_splits=0, indices=None):
    ip, ix, lp = c.get_page_table()
    if indices is None:
        indices = torch.from_numpy(ix).to("cuda")
    out = torch.full_like(q, float("nan"))
    attention_noalloc(q, out, c.pool[0], indices, ip, lp, [w.Nq] * n_streams, c.max_pages, w.P,
                      lse=lse, num_splits=num_splits)
    return out


def _fit_splits(rows, H, D):
    return min(64, SCRATCH_FLOATS // (rows * H * (D + 1)))


@pytest.mark.parametrize("splits", ["auto", "one", "fit"])
@pytest.mark.parametrize("with_lse", [True, False])
@pytest.mark.parametrize("case", ["vitl_bf16", "ragged_fp16_d128"])
def test_noalloc_matches_run_twice(case, with_lse, splits):
    if case == "vitl_bf16":
        w, ages = WORKLOADS["vitl_step"], [90]
    else:
        w, ages = small_workload(H=4, D=128, P=784, ns=6, S=4, W=8, dtype="fp16", R=8), [5, 30]
    c, q, _, _ = _filled(w, ages)
    ns = {"auto": 0, "one": 1, "fit": _fit_splits(q.shape[0], w.H, w.D)}[splits]
    ref_lse = torch.empty((q.shape[0], w.H), dtype=torch.float32, device="cuda")
    ref = c.run(0, q, lse=ref_lse)
    for call in range(2):
        lse = (torch.full((q.shape[0], w.H), float("nan"), dtype=torch.float32, device="cuda")
               if with_lse else None)
        out = _call(c, q, w, len(ages), lse=lse, num_splits=ns)
        torch.cuda.synchronize()
        _close(out, ref)
        if with_lse:
            np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=2e-2)
    noalloc_device_error()


def test_noalloc_ragged_batch_with_a_one_tile_stream_against_oracle():
    """Three streams: one frame old (a single KV tile at D = 64), ten and
    twenty-five frames old.  Automatic and explicit splits, every output
    element against the oracle."""
    w = small_workload(H=2, D=64, P=100, ns=6, S=2, W=6, dtype="bf16", R=25)
    ages = [1, 10, 25]
    c, q, sts, q64 = _filled(w, ages, oracle=True)
    refs = [oracle_out(sts[s], q64[s * w.Nq:(s + 1) * w.Nq])[0] for s in range(3)]
    for ns in (0, 1, 7):
        for call in range(2):
            out = _call(c, q, w, 3, num_splits=ns)
            for s in range(3):
                assert_close(out[s * w.Nq:(s + 1) * w.Nq], refs[s],
                             what=f"splits={ns} call={call} stream={s}")
    noalloc_device_error()


def test_noalloc_against_oracle_full_size_sampled_rows():
    """The ViT-L-sized step (one frame over 72 patch pages and 540 special
    tokens): sampled query rows of every head against the oracle."""
    w = WORKLOADS["vitl_step"]
    c, q, sts, q64 = _filled(w, [90], oracle=True)
    rows = np.array(sorted({0, 1, 5, 127, 128, 700, 1279, 1280, 1374}))
    ref, _ = oracle_out(sts[0], q64, rows)
    for call in range(2):
        out = _call(c, q, w, 1)
        assert_close(out[rows], ref, what=f"call {call}")
    noalloc_device_error()


def test_noalloc_reports_out_of_range_page_id_then_runs_clean():
    """A page id past max_pages in the visible table: the kernel reads page 0
    in its place (no out-of-range access) and records it; the error call
    returns SVT_EDEVICE and clears the word, and the next good call is clean
    and correct."""
    w = small_workload(H=2, D=64, P=64, ns=6, S=1, W=3, dtype="bf16", R=6)
    c, q, _, _ = _filled(w, [5])
    noalloc_device_error()                       # start from a clear word
    ref = c.run(0, q)
    ip, ix, lp = c.get_page_table()
    bad = ix.copy()
    bad[1] = c.max_pages + 7
    out = _call(c, q, w, 1, indices=torch.from_numpy(bad).to("cuda"))
    with pytest.raises(SvtError) as e:
        noalloc_device_error()
    assert e.value.code == _lib.SVT_EDEVICE
    assert "page-id" in str(e.value)
    assert torch.isfinite(out.float()).all()
    out = _call(c, q, w, 1)
    noalloc_device_error()                       # clean
    _close(out, ref)


def test_noalloc_rejects_oversized_split_request():
    w = WORKLOADS["vitl_step"]
    c, q, _, _ = _filled(w, [80])
    ip, ix, lp = c.get_page_table()
    indices = torch.from_numpy(ix).to("cuda")
    out = torch.empty_like(q)
    with pytest.raises(SvtError) as e:
        attention_noalloc(q, out, c.pool[0], indices, ip, lp, [w.Nq], c.max_pages, w.P,
                          num_splits=64)
    assert e.value.code == _lib.SVT_EINVAL
    assert "scratch" in str(e.value)


def test_noalloc_on_a_pool_without_cross_frame_special():
    """A pool whose pages hold a frame's patches followed by its specials
    (page_size + num_special tokens per page): the allocation-free call,
    given that page size, matches svt_run, twice in a row."""
    w = small_workload(H=2, D=64, P=100, ns=6, S=1, W=3, dtype="bf16", R=8)
    c = make_cache(w, w.S + w.W + 1, cross_frame_special=False)
    bank = FrameBank(w, 0, 0, need_oracle=False)
    for t in range(7):
        c.append_frame(0, *bank.device(t)[1:])
        c.evict_frames()
    c.build_visible_page_table()
    c.plan([w.Nq])
    q = bank.device(6)[0]
    ref = c.run(0, q)
    ip, ix, lp = c.get_page_table()
    assert list(lp) == [w.P + w.ns]
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        attention_noalloc(q, out, c.pool[0], torch.from_numpy(ix).to("cuda"), ip, lp, [w.Nq],
                          c.max_pages, c.page_tokens)
        _close(out, ref)
    noalloc_device_error()
