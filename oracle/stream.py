"""Frame-list model of the two-stream streaming KV cache (no pages).

What it restates:
  * Two streams.  Patch tokens of a frame are kept while the frame is a
    scale frame or inside the sliding window; special tokens (6 per frame)
    are kept for every frame, forever.  [P1] § Two-Stream KV Cache Design,
    [P2] § Two-Stream Page Design, [P3] § Two-Stream Design: Patch and
    Special Tokens.
  * Scale frames are the first ``scale_frames`` frames and are never evicted;
    the live window holds the most recent ``sliding_window`` frames after the
    scale frames; after each append the oldest window frames beyond
    ``sliding_window`` are dropped.  [P1] § Sliding-Window Eviction Strategy,
    [P3] § Sliding-Window Eviction Strategy, [P3] FAQ "What distinguishes
    scale frames from window frames".
  * Per frame step: append, then evict, then attend over everything visible,
    the frame's own tokens included.  [P1] § Step-by-Step Streaming
    Inference (steps 2-4).
  * Deferred eviction: a frame appended while eviction is deferred is
    provisional; eviction waits until the frame is accepted
    (``execute_deferred_eviction``) and ``rollback_last_frame`` drops it,
    restoring the previous state.  [P3] § Flow-Based Keyframe Selection and
    its FAQ entry.
  * Cache statistics ``{frame_count, scale_pages, live_pages, free_pages,
    special_tokens}``.  [P3] § Implementation Examples, "Inspecting Cache
    Statistics"; [P4] § Practical Usage Examples.

Readings where the pages are silent:
  * Input rows ``0..num_special-1`` of a frame are the special tokens and
    the remaining rows the patch tokens.
  * While a frame is provisional the window holds up to ``sliding_window+1``
    frames (its eviction has not run yet).
  * Scale frames are the first frames ever accepted; a rolled-back frame never
    counts.
  * The visible order is scale frames' patches, then window patches oldest
    to newest, then all special tokens in frame order ([P4] FAQ "How does the
    paged cache handle variable sequence lengths": scale -> live -> special).
  * ``cross_frame_special=False`` ([P3] § Configuration Parameters: the flag
    retains the special tokens of evicted frames; [P3] § Sliding-Window
    Eviction Strategy, "Special Token Retention"): without retention a
    frame's special tokens are visible exactly while its patch tokens are,
    i.e. for the scale frames and the window frames.  Each visible frame then
    contributes its patch tokens followed by its special tokens, scale frames
    first, window frames oldest to newest ([P3] § The Paged KV-Cache
    Architecture: append_frame places patch tokens first, then special
    tokens).
"""

from __future__ import annotations

import numpy as np

from ._util import as64


def visible_frame_ids(n_frames: int, scale_frames: int, sliding_window: int,
                      provisional: bool, cross_frame_special: bool = True):
    """Frame indices whose tokens are visible after the current step.

    Returns ``(scale_ids, window_ids, special_ids)`` for a stream holding
    ``n_frames`` frames (the provisional one, if any, being the last).
    """
    n, S, W = int(n_frames), int(scale_frames), int(sliding_window)
    scale_ids = list(range(min(n, S)))
    rest = list(range(S, n)) if n > S else []
    w = W + (1 if provisional else 0)
    window_ids = rest[len(rest) - w:] if 0 < w < len(rest) else (rest if w > 0 else [])
    special_ids = list(range(n)) if cross_frame_special else scale_ids + window_ids
    return scale_ids, window_ids, special_ids


def visible_token_count(n_frames, P, ns, S, W, provisional=False,
                        cross_frame_special=True) -> int:
    """min(t,S)*P + min(max(t-S,0), W[+1])*P + ns*t, or, without cross-frame
    special retention, (min(t,S) + min(max(t-S,0), W[+1]))*(P+ns)."""
    t = int(n_frames)
    w = W + (1 if provisional else 0)
    frames = min(t, S) + min(max(t - S, 0), w)
    if not cross_frame_special:
        return frames * (P + ns)
    return frames * P + ns * t


class _Frame:
    __slots__ = ("k_special", "v_special", "k_patch", "v_patch")

    def __init__(self, k, v, ns):
        # Views, not copies: a stream that cycles through a few distinct data
        # frames shares their memory.  Callers must not modify the arrays.
        self.k_special = k[:ns]
        self.v_special = v[:ns]
        self.k_patch = k[ns:]
        self.v_patch = v[ns:]


class FrameStream:
    """One stream of one transformer block: per-frame K/V in Python lists."""

    def __init__(self, patches_per_frame: int, num_special: int,
                 scale_frames: int, sliding_window: int, cross_frame_special: bool = True):
        self.P = int(patches_per_frame)
        self.ns = int(num_special)
        self.S = int(scale_frames)
        self.W = int(sliding_window)
        self.cross_frame_special = bool(cross_frame_special)
        self.frames: list[_Frame] = []
        self.provisional = False

    # -- mutation -------------------------------------------------------
    def append_frame(self, k, v, deferred: bool = False) -> None:
        """Append one frame ``[ns+P, H, D]`` (specials first), then evict
        unless ``deferred``."""
        if self.provisional:
            raise RuntimeError("previous frame is still provisional")
        k = as64(k)
        v = as64(v)
        if k.shape != v.shape or k.shape[0] != self.ns + self.P:
            raise ValueError(f"frame rows must be num_special+P={self.ns + self.P}")
        self.frames.append(_Frame(k, v, self.ns))
        self.provisional = bool(deferred)
        if not deferred:
            self._evict()

    def execute_deferred_eviction(self) -> None:
        if not self.provisional:
            raise RuntimeError("no provisional frame")
        self.provisional = False
        self._evict()

    def rollback_last_frame(self) -> None:
        if not self.provisional:
            raise RuntimeError("no provisional frame")
        self.frames.pop()
        self.provisional = False

    def _evict(self) -> None:
        # Frames that left the window never come back: drop their patch data,
        # and their special data without cross-frame retention (keeps the
        # oracle's memory bounded on long streams).
        _, window, _ = visible_frame_ids(len(self.frames), self.S, self.W, False)
        first_live = window[0] if window else len(self.frames)
        for i in range(self.S, first_live):
            f = self.frames[i]
            if f.k_patch is None:
                continue
            f.k_patch = f.v_patch = None
            if not self.cross_frame_special:
                f.k_special = f.v_special = None

    # -- queries --------------------------------------------------------
    def visible_ids(self):
        return visible_frame_ids(len(self.frames), self.S, self.W, self.provisional,
                                 self.cross_frame_special)

    def visible_kv(self, heads=None):
        """(K, V) of all visible tokens, ``[N, H, D]`` float64, in the order
        scale patches -> window patches -> specials.  ``heads`` (a slice or
        index list) restricts the gather to some heads."""
        scale, window, special = self.visible_ids()
        sel = slice(None) if heads is None else heads
        ks, vs = [], []
        for i in scale + window:
            f = self.frames[i]
            assert f.k_patch is not None, "visible frame lost its patches"
            ks.append(f.k_patch[:, sel])
            vs.append(f.v_patch[:, sel])
            if not self.cross_frame_special:       # the frame's own specials follow
                ks.append(f.k_special[:, sel])
                vs.append(f.v_special[:, sel])
        if self.cross_frame_special:
            for i in special:
                ks.append(self.frames[i].k_special[:, sel])
                vs.append(self.frames[i].v_special[:, sel])
        return np.concatenate(ks, 0), np.concatenate(vs, 0)

    def num_visible_tokens(self) -> int:
        return visible_token_count(len(self.frames), self.P, self.ns, self.S,
                                   self.W, self.provisional, self.cross_frame_special)

    def stats(self, patch_capacity: int) -> dict:
        """Cache statistics of this stream when the pool holds
        ``patch_capacity`` patch pages (one per frame)."""
        scale, window, special = self.visible_ids()
        return {
            "frame_count": len(self.frames),
            "scale_pages": len(scale),
            "live_pages": len(window),
            "free_pages": patch_capacity - len(scale) - len(window),
            "special_tokens": self.ns * len(special),
        }
