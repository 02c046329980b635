"""CPU oracle for per-frame paged KV-cache attention -- TEST INFRASTRUCTURE.

A plain, slow, obviously correct restatement of what the streaming scheme
computes: per-frame K/V held in ordinary Python lists (no pages), the visible
set chosen by frame arithmetic, and softmax(Q K^T / sqrt(D)) V in float64.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the C-ABI library and its Python binding) never imports it and
shares no code with it; both only take their inputs from
``streaming_video_transformer_b200.inputs``.

Sources (web pages on the LingBot-Map streaming scheme, cited by title):
  [P1] "How Paged KV Cache Attention Enables ~20 FPS Streaming Inference in LingBot-Map"
  [P2] "How the Paged KV Cache Attention Mechanism Enables Long Sequence Inference in LingBot-Map"
  [P3] "How LingBot-Map Uses KV Caching for Efficient Streaming Inference"
  [P4] "How FlashInfer's Paged KV Cache Attention Outperforms SDPA Fallback in Streaming Inference"

Pins (tests/test_oracle.py): the hand-worked two-frame example, with and
without cross-frame special retention (tests/golden/two_frame_example.txt),
the cache-statistics example printed in [P3] and [P4]
(tests/golden/cache_stats_example.txt), visible-token counts
(tests/golden/visible_counts.txt), brute-force attention with an explicit
visibility mask, torch's float64 scaled-dot-product attention, closed-form
special cases (uniform and one-hot attention), the visible-token-count
formula, rollback restoring outputs, and the RoPE rotation against a complex
form within its fp32 error bound, with unit vectors giving the fp32 tables
exactly.
"""

from .stream import FrameStream, visible_frame_ids
from .attention import attend, attend_lse
from .rope import rope2d

__all__ = ["FrameStream", "visible_frame_ids", "attend", "attend_lse", "rope2d"]
