"""C-ABI library on the host: symbols, allocator bookkeeping, error paths.

No kernel is launched here: caches are created with ``host_only`` so the
allocator runs without a GPU.  Page tables and statistics are compared bit
for bit with the test-only allocator model (tests/alloc_model.py).
"""
import ctypes
import os
import re

import numpy as np
import pytest

import golden_io
from alloc_model import AllocModel
from streaming_video_transformer_b200 import _lib
from streaming_video_transformer_b200.build import build
from streaming_video_transformer_b200.cache import PagedKVCache, SvtError

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    build()
    yield


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "svt.h")).read()
    return sorted(set(re.findall(r"SVT_API\s+[\w\s\*]+?\b(svt_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    names = _declared_symbols()
    assert len(names) == len(_lib.EXPORTED)
    assert sorted(_lib.EXPORTED) == names
    for n in names:
        assert hasattr(lib, n), n


def _host_cache(**kw):
    args = dict(max_pages=40, page_size=4, H=2, D=64, sliding_window=3, scale_frames=2,
                num_special=3, host_only=True)
    args.update(kw)
    return PagedKVCache(**args)


def _check_against(c, m):
    ip, ix, lp = c.get_page_table()
    mip, mix, mlp = m.table()
    assert list(ip) == mip and list(ix) == mix and list(lp) == mlp
    for s in range(len(m.st)):
        assert c.get_cache_stats(s) == m.stats(s)


@pytest.mark.parametrize("cross", [True, False])
@pytest.mark.parametrize("seed", range(6))
def test_random_op_sequences_match_model(seed, cross):
    rng = np.random.default_rng(seed)
    ns_ = int(rng.integers(1, 4))
    P, ns, S, W = int(rng.integers(3, 7)), int(rng.integers(0, 4)), int(rng.integers(0, 3)), int(rng.integers(0, 4))
    ns = min(ns, P)
    max_pages = ns_ * (S + W + 1) + (30 if cross else 0)
    c = _host_cache(max_pages=max_pages, page_size=P, num_special=ns, scale_frames=S,
                    sliding_window=W, num_streams=ns_, num_blocks=2, cross_frame_special=cross)
    m = AllocModel(max_pages, P, ns, S, W, ns_, cross_frame_special=cross)
    for step in range(120):
        s = int(rng.integers(0, ns_))
        st = m.st[s]
        if st.prov is not None:
            if rng.random() < 0.5:
                c.rollback_last_frame(s); m.rollback(s)
            else:
                c.execute_deferred_eviction(s); m.accept(s)
        else:
            defer = rng.random() < 0.3
            c.set_defer_eviction(defer, s); st.defer = defer
            try:
                m_page = m.append(s)
            except MemoryError:
                with pytest.raises(SvtError) as e:
                    c.append_frame(0, stream=s)
                assert e.value.code == _lib.SVT_ENOPAGES
                _check_against(c, m)
                break
            c.append_frame(0, stream=s)
            c.append_frame(1, stream=s)
            c.evict_frames(s); m.evict(s)
        _check_against(c, m)


def test_cache_stats_example_from_pages():
    g = golden_io.kv_file("cache_stats_example.txt")
    c = _host_cache(max_pages=g["patch_capacity"] + 60, page_size=256, num_special=g["num_special"],
                    scale_frames=g["scale_frames"], sliding_window=g["sliding_window"],
                    patch_pages=g["patch_capacity"])
    for _ in range(g["frame_count"]):
        c.append_frame(0)
        c.evict_frames()
    s = c.get_cache_stats()
    for key in ("frame_count", "scale_pages", "live_pages", "free_pages", "special_tokens"):
        assert s[key] == g[key], key


def test_two_frame_example_page_table():
    _, tables = golden_io.two_frame_cases()
    (S, W, t, idx, lpl), = tables
    c = _host_cache(max_pages=12, page_size=2, num_special=1, scale_frames=S, sliding_window=W)
    for _ in range(t):
        c.append_frame(0)
        c.evict_frames()
    ip, ix, lp = c.get_page_table()
    npatch = c.patch_pages
    assert list(ix) == [npatch if x == "NPATCH" else int(x) for x in idx]
    assert list(lp) == [lpl]


def test_two_frame_example_page_table_without_cross_frame_special():
    _, tables = golden_io.two_frame_cases(cross_frame_special=False)
    (S, W, t, idx, lpl), = tables
    c = _host_cache(max_pages=12, page_size=2, num_special=1, scale_frames=S, sliding_window=W,
                    cross_frame_special=False)
    for _ in range(t):
        c.append_frame(0)
        c.evict_frames()
    ip, ix, lp = c.get_page_table()
    assert list(ix) == [int(x) for x in idx]
    assert list(lp) == [lpl]


def test_no_cross_frame_special_counts_and_pool_size():
    """Without retention: the tiny stream's visible counts (golden), the
    special-token statistic (the specials of resident frames only), a pool
    with no special pages at all, and pool pages of page_size + num_special
    tokens."""
    vc = golden_io.visible_counts()
    counts = [int(x) for x in vc["tiny_nocross"][1]]
    P, ns, S, W = 16, 6, 2, 4
    c = _host_cache(max_pages=S + W + 1, page_size=P, num_special=ns, scale_frames=S,
                    sliding_window=W, cross_frame_special=False)
    for t in range(1, 13):
        c.append_frame(0)
        c.evict_frames()
        ip, ix, lp = c.get_page_table()
        assert (len(ix) - 1) * (P + ns) + lp[0] == counts[t - 1]
        st = c.get_cache_stats()
        assert st["special_tokens"] == ns * (st["scale_pages"] + st["live_pages"])
    with pytest.raises(SvtError):                            # cross retention needs special pages
        _host_cache(max_pages=S + W + 1, page_size=P, num_special=ns, scale_frames=S,
                    sliding_window=W)
    lib = _lib.load()
    opts = _lib.CacheOpts()
    lib.svt_default_opts(ctypes.byref(opts))
    assert opts.no_cross_frame_special == 0
    opts.num_special = ns
    base = lib.svt_pool_bytes(10, P, 2, 64, ctypes.byref(opts))
    opts.no_cross_frame_special = 1
    assert lib.svt_pool_bytes(10, P, 2, 64, ctypes.byref(opts)) == base * (P + ns) // P


def test_steady_state_page_counts():
    vc = golden_io.visible_counts()
    c = _host_cache(max_pages=8 + 64 + 1 + 10, page_size=1369, num_special=6, scale_frames=8,
                    sliding_window=64)
    for _ in range(200):
        c.append_frame(0)
        c.evict_frames()
    ip, ix, lp = c.get_page_table()
    body = dict(tok.split("=") for tok in vc["vitl_pages"][1])
    assert len(ix) == int(body["patch_pages"]) + int(body["special_pages"])
    assert lp[0] == int(body["last_page_len"])
    assert (len(ix) - 1) * 1369 + lp[0] == int(vc["vitl"][1][0])


def test_rollback_restores_allocator_exactly():
    c = _host_cache(max_pages=30, page_size=4, num_special=3, scale_frames=1, sliding_window=2)
    for _ in range(5):
        c.append_frame(0); c.evict_frames()
    before = (c.get_page_table(), c.get_cache_stats())
    c.set_defer_eviction(True)
    c.append_frame(0)
    c.evict_frames()                      # no-op while provisional
    assert c.get_cache_stats()["live_pages"] == 3
    c.rollback_last_frame()
    after = (c.get_page_table(), c.get_cache_stats())
    for a, b in zip(before[0], after[0]):
        assert np.array_equal(a, b)
    assert before[1] == after[1]
    # the next frame gets the page the rolled-back one had
    c.set_defer_eviction(False)
    c.append_frame(0)
    assert c.get_page_table()[1][c.get_cache_stats()["scale_pages"] + 2] >= 0


def test_error_paths():
    c = _host_cache(max_pages=9, page_size=4, num_special=3, scale_frames=1, sliding_window=1,
                    num_blocks=2)
    with pytest.raises(SvtError) as e:
        c.rollback_last_frame()
    assert e.value.code == _lib.SVT_ESTATE
    with pytest.raises(SvtError) as e:
        c.execute_deferred_eviction()
    assert e.value.code == _lib.SVT_ESTATE
    with pytest.raises(SvtError) as e:
        c.append_frame(1)                 # block 1 before block 0
    assert e.value.code == _lib.SVT_ESTATE
    c.append_frame(0)
    with pytest.raises(SvtError) as e:
        c.append_frame(0)                 # block 1 missing
    assert e.value.code == _lib.SVT_ESTATE
    c.append_frame(1)
    c.append_frame(0); c.append_frame(1)  # scale 1, window 1
    c.append_frame(0); c.append_frame(1)  # window 2 > W=1 now (no evict)
    with pytest.raises(SvtError) as e:
        c.append_frame(0)                 # forgot evict
    assert e.value.code == _lib.SVT_ESTATE
    c.evict_frames()
    with pytest.raises(SvtError) as e:
        c.plan([100])                     # table not built since the change
    assert e.value.code == _lib.SVT_ESTATE
    c.build_visible_page_table()
    c.plan([7])
    with pytest.raises(SvtError) as e:
        c.append_frame(5)
    assert e.value.code == _lib.SVT_EINVAL
    with pytest.raises(SvtError) as e:
        c.append_frame(0, stream=1)
    assert e.value.code == _lib.SVT_EINVAL
    # pool of 3 patch pages (1+1+1) and 6 special pages: specials run out after 8 frames
    for _ in range(20):
        try:
            c.append_frame(0); c.append_frame(1); c.evict_frames()
        except SvtError as err:
            assert err.code == _lib.SVT_ENOPAGES
            break
    else:
        pytest.fail("pool never ran out")


def test_create_validation():
    with pytest.raises(SvtError):
        _host_cache(num_special=9, page_size=4)              # specials > page
    with pytest.raises(SvtError):
        _host_cache(max_pages=5)                             # patch pages need S+W+1=6
    with pytest.raises(SvtError):
        _host_cache(page_size=16, rope_grid=3)               # 3*3 != 16
    lib = _lib.load()                                        # device cache without a pool
    opts = _lib.CacheOpts()
    lib.svt_default_opts(ctypes.byref(opts))
    opts.num_special = 3
    h = ctypes.c_void_p(0)
    assert lib.svt_create_cache(40, 4, 2, 64, 3, 2, ctypes.byref(opts), ctypes.byref(h)) == _lib.SVT_EINVAL
    assert b"pool" in lib.svt_last_error()


def test_set_free_lists_permutes_ids():
    c = _host_cache(max_pages=14, page_size=4, num_special=3, scale_frames=1, sliding_window=2)
    npatch = c.patch_pages
    perm_p = list(reversed(range(npatch)))
    perm_s = list(reversed(range(npatch, 14)))
    c.set_free_lists(perm_p, perm_s)
    c.append_frame(0); c.evict_frames()
    ip, ix, lp = c.get_page_table()
    assert list(ix) == [perm_p[0], perm_s[0]]
    with pytest.raises(SvtError):
        c.set_free_lists(perm_p, perm_s)                    # not empty any more
    c.reset()
    assert c.get_cache_stats()["frame_count"] == 0


@pytest.mark.parametrize("D,tile", [(64, 128), (128, 64)])
def test_plan_tiles_items_and_split_bounds(D, tile):
    """The plan's work decomposition: KV tiles per stream are whole pages of
    ceil(page_size / tile) tiles plus ceil(last_page_len / tile) (the kernel
    reads 128-token tiles at D = 64 and 64-token tiles at D = 128), one work
    item per (head, 128-row query tile, KV chunk), and a chunk count between
    1 and max_splits that never exceeds the stream's tile count."""
    P, ns, S, W, H = 100, 6, 2, 3, 4
    ages = (1, 4, 9)
    qo = [P + ns, 2 * (P + ns), 5]
    c = _host_cache(max_pages=3 * (S + W + 1) + 8, page_size=P, H=H, D=D, sliding_window=W,
                    scale_frames=S, num_special=ns, num_streams=len(ages), max_splits=8,
                    max_qo_len=sum(qo))
    for s, age in enumerate(ages):
        for _ in range(age):
            c.append_frame(0, stream=s)
            c.evict_frames(s)
    c.build_visible_page_table()
    c.plan(qo)
    info = c.plan_info()
    ip, ix, lp = c.get_page_table()
    items = 0
    for s, age in enumerate(ages):
        n_pages = ip[s + 1] - ip[s]
        tiles = (n_pages - 1) * -(-P // tile) + -(-int(lp[s]) // tile)
        assert info["kv_tiles"][s] == tiles
        assert info["kv_tokens"][s] == (n_pages - 1) * P + int(lp[s])
        assert info["kv_tokens"][s] == min(age, S) * P + min(max(age - S, 0), W) * P + ns * age
        assert 1 <= info["splits"][s] <= min(8, tiles)
        items += H * -(-qo[s] // 128) * info["splits"][s]
    assert info["num_items"] == items


def test_binding_constants_match_the_header():
    """The binding's copies of the header's constants (status codes, dtypes,
    the stream limit that sizes svt_plan_info's arrays)."""
    import re
    hdr = open(os.path.join(ROOT, "include", "svt.h")).read()
    m = re.search(r"#define SVT_MAX_STREAMS (\d+)", hdr)
    assert m and int(m.group(1)) == _lib.MAX_STREAMS
    for name in ("SVT_OK", "SVT_EINVAL", "SVT_ENOPAGES", "SVT_ESTATE", "SVT_ECUDA", "SVT_EDEVICE",
                 "SVT_BF16", "SVT_FP16", "SVT_FP32"):
        m = re.search(name + r"\s*=\s*(-?\d+)", hdr)
        assert m, name
        assert int(m.group(1)) == getattr(_lib, name), name
