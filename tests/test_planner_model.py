"""The host planner's split choice against its cost model searched in full.

svt_plan picks, per frame step, how many KV chunks each stream's work is cut
into.  Its model: a work item is one 128-row query tile of one head over one
KV chunk and costs a fixed 2 us plus its KV tiles at a fixed rate; items are
list-scheduled, in launch order, onto the CTA slots (148 SMs x 2); a split
adds the merge's fixed and per-byte cost; candidate k (1..max_splits) scales
every stream's chunk count with its tile count, and a later k replaces the
best only if it is more than 2% faster.  The library stops the search once
a lower bound of the model rules out every larger k.  Here the model is
restated in Python and searched over every k, and the library's choice must
be the same on random host-only caches (no GPU)."""
import heapq
import math

import numpy as np
import pytest

from streaming_video_transformer_b200.cache import PagedKVCache

SLOTS = 148 * 2
TILE_M = 128


def model_splits(qo, tiles, H, D, max_splits):
    TN = 128 if D == 64 else 64
    tile_us = 4.0 * TILE_M * TN * D / 6.6e6 * 2
    item_us = 2.0
    max_tiles = max([t for q, t in zip(qo, tiles) if q] or [0])
    qt = [-(-q // TILE_M) for q in qo]
    best, best_t = [1] * len(qo), math.inf
    for k in range(1, max_splits + 1):
        ch, costs, merge_bytes, split = [1] * len(qo), [], 0.0, False
        for i, (q, t) in enumerate(zip(qo, tiles)):
            if not q:
                continue
            cc = math.ceil(k * t / max(1, max_tiles))
            cc = max(1, min(cc, max_splits, t))
            ch[i] = cc
            if cc > 1:
                split = True
                merge_bytes += q * H * (D + 1) * 4.0 * (cc + 1)
            for _ in range(H):
                for cix in range(cc):
                    t0, t1 = cix * t // cc, (cix + 1) * t // cc
                    costs += [item_us + (t1 - t0) * tile_us] * qt[i]
        slots = [0.0] * SLOTS
        end = 0.0
        for c in costs:
            s = heapq.heappop(slots) + c
            end = max(end, s)
            heapq.heappush(slots, s)
        total = end + (4.0 + merge_bytes / 5.0e6 if split else 0.0)
        if total < best_t * 0.98:
            best_t, best = total, ch
    return [b if q else 0 for b, q in zip(best, qo)]


def _cache(rng):
    H = int(rng.choice([2, 4, 8, 16]))
    D = int(rng.choice([64, 128]))
    P = int(rng.choice([16, 100, 256, 784, 1369]))
    S, W, ns = int(rng.integers(0, 9)), int(rng.integers(1, 65)), 6
    n = int(rng.integers(1, 5))
    ages = [int(rng.integers(1, 300)) for _ in range(n)]
    cross = bool(rng.random() < 0.7)
    max_splits = int(rng.choice([4, 8, 16]))
    mp = n * (S + W + 1) + sum(-(-a * ns // P) for a in ages) + 4 * n
    c = PagedKVCache(mp, P, H, D, W, S, num_special=ns, num_streams=n, host_only=True,
                     max_qo_len=n * 8 * (P + ns), max_splits=max_splits,
                     cross_frame_special=cross)
    for s, a in enumerate(ages):
        for _ in range(a):
            c.append_frame(0, stream=s)
            c.evict_frames(s)
    c.build_visible_page_table()
    return c, H, D, max_splits


@pytest.mark.parametrize("seed", range(24))
def test_planner_matches_full_model_search(seed):
    rng = np.random.default_rng(seed)
    c, H, D, max_splits = _cache(rng)
    n = c.num_streams
    ip, _, lp = c.get_page_table()
    TN = 128 if D == 64 else 64
    tpp = -(-c.page_tokens // TN)
    qo = [int(rng.choice([0, 1, 40, c.page_size + 6, 3 * (c.page_size + 6)])) for _ in range(n)]
    if not any(qo):
        qo[0] = c.page_size + 6
    extra = [int(rng.choice([0, c.page_size + 6])) if q else 0 for q in qo]
    for xl in (None, extra):
        tiles = []
        for i in range(n):
            npg = int(ip[i + 1] - ip[i])
            t = ((npg - 1) * tpp + -(-int(lp[i]) // TN)) if npg else 0
            tiles.append(t + (-(-xl[i] // TN) if xl else 0))
        c.plan(qo, extra_len=xl)
        info = c.plan_info()
        assert info["kv_tiles"] == tiles
        assert info["splits"] == model_splits(qo, tiles, H, D, max_splits), (qo, tiles, xl)
    c.close()
