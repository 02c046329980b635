"""2-D rotary position embedding on the patch rows of a frame.

The pages say only that query and key are prepared with an optional RoPE
before the key/value are appended ([P1] § Step-by-Step Streaming Inference,
step 1).  The 2-D convention used here is a reading of that silence:

  * patch p (0-based among the patch rows, raster order) sits at grid row
    r = p // grid and column c = p % grid; special rows are not rotated;
  * each head's D features are split in two halves of m = D/2; the first
    half is rotated by position r, the second by position c;
  * inside a half, feature i pairs with feature i + m/2 (rotate-half form),
    angle = pos * theta ** (-2 i / m) for i < m/2:
        (a, b) -> (a cos - b sin, a sin + b cos).

Computed in float64; the caller rounds to the storage dtype.
"""

from __future__ import annotations

import numpy as np

from ._util import as64


def rope2d(x, num_special: int, grid: int, theta: float):
    """Rotate the patch rows of ``x [ns+grid*grid, H, D]``; returns float64."""
    x = as64(x).copy()
    n, H, D = x.shape
    if n != num_special + grid * grid:
        raise ValueError("rows must be num_special + grid*grid")
    if D % 4:
        raise ValueError("D must be a multiple of 4")
    m = D // 2
    half = m // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / m)                       # [half]
    p = np.arange(grid * grid)
    for sect, pos in ((0, p // grid), (1, p % grid)):
        ang = pos[:, None].astype(np.float64) * inv_freq[None, :]   # [P, half]
        c = np.cos(ang)[:, None, :]
        s = np.sin(ang)[:, None, :]
        lo = slice(sect * m, sect * m + half)
        hi = slice(sect * m + half, sect * m + m)
        a = x[num_special:, :, lo].copy()
        b = x[num_special:, :, hi].copy()
        x[num_special:, :, lo] = a * c - b * s
        x[num_special:, :, hi] = a * s + b * c
    return x
