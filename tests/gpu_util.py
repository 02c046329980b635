"""Helpers shared by the GPU parity tests: drive the library and the oracle
on the same seeded inputs and compare."""
from __future__ import annotations

import numpy as np
import torch

from oracle import FrameStream, attend_lse, rope2d
from streaming_video_transformer_b200.cache import PagedKVCache
from streaming_video_transformer_b200.inputs import frame_qkv

# Tolerances: bf16/fp16 storage, fp32 accumulation (max-abs and relative L2),
# and the fp32-FMA path.
TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 5e-3
TOL_FP32_REL_L2 = 1e-5


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close(gpu, ref, fp32=False, what="", fp32_tol=TOL_FP32_REL_L2):
    g = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    r = rel_l2(g, ref)
    if fp32:
        assert r <= fp32_tol, f"{what}: rel-L2 {r:.3e} > {fp32_tol:.3e}"
    else:
        mx = float(np.max(np.abs(g - ref)))
        assert mx <= TOL_MAX_ABS, f"{what}: max-abs {mx:.3e} > {TOL_MAX_ABS}"
        assert r <= TOL_REL_L2, f"{what}: rel-L2 {r:.3e} > {TOL_REL_L2}"
    return r


def max_pages_for(w, frames_per_stream, num_streams=1, slack=2):
    """Patch pages S+W+1 per stream plus the special pages the streams need."""
    need_sp = sum(-(-f * w.ns // w.P) for f in frames_per_stream) + slack * num_streams
    return num_streams * (w.S + w.W + 1) + need_sp


def make_cache(w, max_pages, num_streams=1, **kw):
    return PagedKVCache(max_pages, w.P, w.H, w.D, w.W, w.S, num_blocks=w.blocks,
                        num_special=w.ns, num_streams=num_streams, dtype=w.dtype,
                        rope_grid=w.rope_grid, rope_theta=w.rope_theta, **kw)


def oracle_stream_for(cache, w):
    """The oracle stream matching a cache's special-token retention."""
    return FrameStream(w.P, w.ns, w.S, w.W, cross_frame_special=cache.cross_frame_special)


class FrameBank:
    """The R distinct data frames of (block, stream), on the device and as
    float64 oracle inputs (with RoPE applied to the patch rows of Q and K
    and rounded to the storage dtype, when the workload has RoPE)."""

    def __init__(self, w, block, stream, device="cuda", need_oracle=True):
        self.w = w
        self.dev, self.o = [], []
        for i in range(w.R):
            q, k, v = frame_qkv(w, block, stream, i)
            self.dev.append(tuple(x.to(device) for x in (q, k, v)))
            if need_oracle:
                if w.rope_grid:
                    qo = torch.from_numpy(rope2d(q, w.ns, w.rope_grid, w.rope_theta)).to(q.dtype)
                    ko = torch.from_numpy(rope2d(k, w.ns, w.rope_grid, w.rope_theta)).to(k.dtype)
                else:
                    qo, ko = q, k
                self.o.append(tuple(x.double().numpy() for x in (qo, ko, v)))

    def device(self, t):
        return self.dev[t % self.w.R]

    def oracle(self, t):
        return self.o[t % self.w.R]


def oracle_stream(w):
    return FrameStream(w.P, w.ns, w.S, w.W)


def oracle_out(st, q64, rows=None):
    k, v = st.visible_kv()
    qs = q64 if rows is None else q64[rows]
    return attend_lse(qs, k, v)


def gather_visible(cache, block, stream, dev_table=True):
    """K and V of a stream's visible tokens read from the pool through the
    (device or host) page table, float64 numpy [N, H, D]."""
    ip, ix, lp = cache.read_device_page_table() if dev_table else cache.get_page_table()
    pages = ix[ip[stream]:ip[stream + 1]]
    pool = cache.pool[block]                                  # [max_pages, 2, P, H, D]
    sel = pool[torch.as_tensor(pages, dtype=torch.long, device=pool.device)]
    n = len(pages)
    k = sel[:, 0].reshape(n * cache.page_tokens, cache.H, cache.D)
    v = sel[:, 1].reshape(n * cache.page_tokens, cache.H, cache.D)
    ntok = (n - 1) * cache.page_tokens + int(lp[stream])
    return k[:ntok].double().cpu().numpy(), v[:ntok].double().cpu().numpy()
