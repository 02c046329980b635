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


def rope2d_fused_fp32(x, num_special, grid, theta):
    """The 2-D RoPE rotation (patch row/column positions, rotate-half pairs)
    evaluated in fp32, each output one fused multiply-add over the other
    product rounded to fp32 (the way an FMA unit evaluates a*c - b*s).  Like the float64 rotation it is a valid
    evaluation of the same formula; rounded to a 16-bit storage type, the two
    can differ by one step on a rare element.  Tests use the spread between
    the oracle run on each to size the fp32 path's bound on RoPE workloads.
    Returns float64 [ns+grid*grid, H, D]."""
    x = np.asarray(x.float().numpy() if hasattr(x, "float") else x, np.float32).copy()
    D = x.shape[2]
    m, half = D // 2, D // 4
    inv_freq = theta ** (-2.0 * np.arange(half, dtype=np.float64) / m)
    p = np.arange(grid * grid)
    for sect, pos in ((0, p // grid), (1, p % grid)):
        ang = pos[:, None].astype(np.float64) * inv_freq[None, :]
        c = np.cos(ang).astype(np.float32)[:, None, :]
        s = np.sin(ang).astype(np.float32)[:, None, :]
        lo = slice(sect * m, sect * m + half)
        hi = slice(sect * m + half, sect * m + m)
        a = x[num_special:, :, lo].copy()
        b = x[num_special:, :, hi].copy()
        bs = (b * s).astype(np.float32).astype(np.float64)
        bc = (b * c).astype(np.float32).astype(np.float64)
        # a*c and a*s are exact in float64 (24 x 24 bits); one final rounding.
        x[num_special:, :, lo] = (a.astype(np.float64) * c - bs).astype(np.float32)
        x[num_special:, :, hi] = (a.astype(np.float64) * s + bc).astype(np.float32)
    return x.astype(np.float64)


def max_pages_for(w, frames_per_stream, num_streams=1, slack=2):
    """Patch pages S+W+1 per stream plus the special pages the streams need."""
    need_sp = sum(-(-f * w.ns // w.P) for f in frames_per_stream) + slack * num_streams
    return num_streams * (w.S + w.W + 1) + need_sp


def make_cache(w, max_pages, num_streams=1, **kw):
    return PagedKVCache(max_pages, w.P, w.H, w.D, w.W, w.S, num_blocks=w.blocks,
                        num_special=w.ns, num_streams=num_streams, dtype=w.dtype,
                        rope_grid=w.rope_grid, rope_theta=w.rope_theta, **kw)


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
    k = sel[:, 0].reshape(n * cache.page_size, cache.H, cache.D)
    v = sel[:, 1].reshape(n * cache.page_size, cache.H, cache.D)
    ntok = (n - 1) * cache.page_size + int(lp[stream])
    return k[:ntok].double().cpu().numpy(), v[:ntok].double().cpu().numpy()
