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

Precision (also a reading: the pages fix none).  The rotation is one stated
fp32 computation, so that every correct implementation produces the same
bits:
  * cs = fp32(cos(angle)), sn = fp32(sin(angle)), the angle and both
    functions evaluated in float64 and each rounded once to fp32;
  * the input values are taken in fp32 (bf16, fp16 and fp32 storage values
    are exact there);
  * a' = rn(rn(a*cs) - rn(b*sn)),  b' = rn(rn(a*sn) + rn(b*cs)),
    every product, difference and sum rounded to fp32 (round to nearest
    even), with no fused multiply-add;
  * the caller rounds a', b' once more, to the storage dtype.
"""

from __future__ import annotations

import numpy as np

from ._util import as64


def rope_tables(grid: int, D: int, theta: float):
    """``(cs, sn)``, each float32 ``[grid, D//4]``: the fp32 cosine and sine of
    ``pos * theta ** (-2 i / m)`` for positions ``0..grid-1`` and ``i < m/2``."""
    m = D // 2
    half = m // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = float(theta) ** (-2.0 * i / m)                          # [half]
    ang = np.arange(grid, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope2d(x, num_special: int, grid: int, theta: float):
    """Rotate the patch rows of ``x [ns+grid*grid, H, D]``.

    Returns float32 numpy ``[ns+grid*grid, H, D]`` (the fp32 results of the
    formula in the module docstring, before the final rounding to storage).
    """
    x = as64(x).astype(np.float32)
    n, H, D = x.shape
    if n != num_special + grid * grid:
        raise ValueError("rows must be num_special + grid*grid")
    if D % 4:
        raise ValueError("D must be a multiple of 4")
    m = D // 2
    half = m // 2
    cs_tab, sn_tab = rope_tables(grid, D, theta)
    out = x.copy()
    p = np.arange(grid * grid)
    for sect, pos in ((0, p // grid), (1, p % grid)):
        cs = cs_tab[pos][:, None, :]                                   # [P, 1, half]
        sn = sn_tab[pos][:, None, :]
        lo = slice(sect * m, sect * m + half)
        hi = slice(sect * m + half, sect * m + m)
        a = x[num_special:, :, lo]
        b = x[num_special:, :, hi]
        # numpy float32 arithmetic: each operation is rounded to fp32 on its own
        ac = np.multiply(a, cs, dtype=np.float32)
        bs = np.multiply(b, sn, dtype=np.float32)
        as_ = np.multiply(a, sn, dtype=np.float32)
        bc = np.multiply(b, cs, dtype=np.float32)
        out[num_special:, :, lo] = np.subtract(ac, bs, dtype=np.float32)
        out[num_special:, :, hi] = np.add(as_, bc, dtype=np.float32)
    return out
