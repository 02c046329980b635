"""Dense softmax attention in float64 over the visible tokens.

For each query row i and head h:
    s_ij = (q_i . k_j) / sqrt(D)
    O[i,h,:] = sum_j exp(s_ij - m_i) v_j / sum_j exp(s_ij - m_i),  m_i = max_j s_ij
    LSE[i,h] = m_i + log(sum_j exp(s_ij - m_i))      (natural log)

There is no causal mask: a frame's queries attend to every visible token,
their own frame's included ([P1] § Step-by-Step Streaming Inference, step 4;
[P2] § FlashInfer Kernel Execution).  The upstream validates its fused kernel
by gathering the paged K/V into dense tensors and running dense attention in
fp32 ([P2] § Memory Efficiency Analysis, force_fp32); this is that dense
computation, in float64, from the stored (already rounded) input values.
"""

from __future__ import annotations

import numpy as np

from ._util import as64


def attend_lse(q, k, v, row_block: int = 256):
    """Return ``(O, LSE)``: ``O [Nq,H,D]`` and ``LSE [Nq,H]`` in float64."""
    q, k, v = as64(q), as64(k), as64(v)
    nq, H, D = q.shape
    n = k.shape[0]
    if k.shape != (n, H, D) or v.shape != (n, H, D):
        raise ValueError("q, k, v must be [N, H, D] with matching H, D")
    if n == 0:
        raise ValueError("no visible tokens")
    scale = 1.0 / np.sqrt(D)
    o = np.empty((nq, H, D), dtype=np.float64)
    lse = np.empty((nq, H), dtype=np.float64)
    for h in range(H):
        kh = np.ascontiguousarray(k[:, h, :])
        vh = np.ascontiguousarray(v[:, h, :])
        for r0 in range(0, nq, row_block):
            qh = q[r0:r0 + row_block, h, :]
            s = (qh @ kh.T) * scale
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            den = e.sum(axis=1, keepdims=True)
            o[r0:r0 + row_block, h, :] = (e @ vh) / den
            lse[r0:r0 + row_block, h] = (m + np.log(den))[:, 0]
    return o, lse


def attend(q, k, v):
    """``O [Nq,H,D]`` float64 (see module docstring)."""
    return attend_lse(q, k, v)[0]
