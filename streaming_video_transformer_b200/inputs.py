"""Seeded synthetic inputs for the streaming paged-attention workloads.

This module only draws random numbers and names workload shapes.  It holds
none of the caching or attention arithmetic, so that the CPU oracle and the
CUDA path can both take their inputs from it without sharing any of the
method's code.

Recipe (every workload):
  * One frame = ``Nq = num_special + patches_per_frame`` token rows.  Rows
    ``0 .. num_special-1`` are the special tokens (camera / register / scale
    tokens), rows ``num_special ..`` are the patch tokens in raster order of
    the patch grid.
  * Q, K, V of frame data index ``i`` for (block ``b``, stream ``s``) are drawn
    N(0, 1) in float32 from a ``torch.Generator`` seeded with
    ``frame_seed(seed, b, s, i)``, multiplied by ``data_scale`` and rounded
    once to the storage dtype.
  * A stream of ``T`` frames cycles through ``R`` distinct data frames: frame
    ``t`` uses data index ``t % R`` (``R >= T`` gives all-distinct frames).
  * Keyframe accept/reject decisions for the rollback workload are drawn with
    ``numpy.random.default_rng(seed).random() < reject_p`` once per deferred
    frame, in stream order.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


@dataclass(frozen=True)
class Workload:
    name: str
    H: int                      # attention heads
    D: int                      # head dim
    P: int                      # patches per frame == page_size
    ns: int                     # special tokens per frame
    S: int                      # scale frames
    W: int                      # sliding window (frames)
    dtype: str                  # storage dtype of Q/K/V and the pool
    seed: int
    blocks: int = 1             # transformer blocks (one pool region each)
    frames: int = 1             # frames streamed (per stream)
    ages: tuple = ()            # batched streams: frames already in each stream
    R: int = 16                 # distinct data frames per (block, stream)
    data_scale: float = 1.0
    rope_grid: int = 0          # 0 = no RoPE, else side of the square patch grid
    rope_theta: float = 100.0
    defer_every: int = 0        # every n-th offered frame is deferred (0 = never)
    reject_p: float = 0.0
    note: str = field(default="", compare=False)

    @property
    def Nq(self) -> int:
        return self.P + self.ns

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]


# Shapes of the pages' workload: a ViT-L/14 on 518 px frames (37 x 37 = 1369
# patches), 16 heads of 64, 6 special tokens, window 64, scale frames 8.
WORKLOADS = {
    "tiny_stream": Workload(
        "tiny_stream", H=2, D=64, P=16, ns=6, S=2, W=4, dtype="bf16", seed=1001,
        frames=12, R=12,
        note="1 block, 12 frames one at a time, all frames distinct"),
    "vitl_step": Workload(
        "vitl_step", H=16, D=64, P=1369, ns=6, S=8, W=64, dtype="bf16", seed=1002,
        frames=201, R=16, data_scale=1.0 / math.sqrt(64),
        note="cache pre-filled with 200 frames, one 1375-token frame attends"),
    "vitl_stream24": Workload(
        "vitl_stream24", H=16, D=64, P=1369, ns=6, S=8, W=64, dtype="bf16", seed=1003,
        blocks=24, frames=1000, R=16, rope_grid=37, rope_theta=100.0,
        note="24 blocks, 1000 frames, 2-D RoPE on patch Q/K"),
    "ragged4": Workload(
        "ragged4", H=8, D=128, P=784, ns=6, S=4, W=32, dtype="fp16", seed=1004,
        ages=(10, 70, 300, 2000), R=16,
        note="4 streams of different ages in one pool, one batched run"),
    "rollback10k": Workload(
        "rollback10k", H=16, D=64, P=1369, ns=6, S=8, W=64, dtype="bf16", seed=1005,
        frames=10000, R=16, defer_every=3, reject_p=0.3,
        note="every 3rd frame deferred, rejected with p=0.3"),
}


def frame_seed(seed: int, block: int, stream: int, data_index: int) -> int:
    """Counter-style seed for one data frame (disjoint bit fields)."""
    assert 0 <= data_index < (1 << 20) and 0 <= stream < (1 << 8) and 0 <= block < (1 << 12)
    return (int(seed) << 40) | (block << 28) | (stream << 20) | data_index


def frame_qkv(w: Workload, block: int, stream: int, frame: int, dtype=None):
    """Q, K, V of one frame as CPU tensors ``[Nq, H, D]`` in the storage dtype."""
    dt = DTYPES[dtype] if isinstance(dtype, str) else (dtype or w.torch_dtype)
    g = torch.Generator().manual_seed(frame_seed(w.seed, block, stream, frame % w.R))
    out = []
    for _ in range(3):
        x = torch.randn((w.Nq, w.H, w.D), generator=g, dtype=torch.float32)
        if w.data_scale != 1.0:
            x = x * w.data_scale
        out.append(x.to(dt).contiguous())
    return tuple(out)


def keyframe_decisions(w: Workload, n_offered: int):
    """Per offered frame: (deferred, rejected).  Frames with ``t % defer_every
    == defer_every - 1`` are deferred; each deferred frame is rejected iff the
    next draw of ``default_rng(seed)`` is below ``reject_p``."""
    rng = np.random.default_rng(w.seed)
    out = []
    for t in range(n_offered):
        deferred = w.defer_every > 0 and (t % w.defer_every) == w.defer_every - 1
        rejected = bool(rng.random() < w.reject_p) if deferred else False
        out.append((deferred, rejected))
    return out


def small_workload(**kw) -> Workload:
    """An ad-hoc workload for tests (same recipe, caller-chosen shape)."""
    base = dict(H=2, D=64, P=16, ns=6, S=2, W=4, dtype="bf16", seed=77, frames=8, R=64)
    base.update(kw)
    name = base.pop("name", "adhoc")
    return Workload(name, **base)
