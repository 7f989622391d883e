"""The pages' blockwise online-softmax merge, in float64 numpy.

TEST INFRASTRUCTURE ONLY (see the package docstring). This routine is not the oracle the
CUDA path is compared with; it exists so the tests can check the pages' claim that the
blockwise merge reproduces the full softmax exactly (up to rounding).

Page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下", section "分块计算，这事没那么简单":
each block keeps two statistics, its maximum m and its sum term d; a new block updates
m and d and corrects the results of the earlier blocks; joined together the result equals
the standard softmax. Written out (the page states this in prose only): for a new block
of scores s with values v,
    m_new = max(m, max(s))
    d     = d * exp(m - m_new) + sum(exp(s - m_new))
    acc   = acc * exp(m - m_new) + sum(exp(s - m_new) * v)
and at the end out = acc / d, lse = m + ln d.
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def online_softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, block: int,
                             scale: Optional[float] = None, causal: bool = False):
    """Single-head attention (q (Sq, D), k/v (Sk, D)) by blockwise merging over key blocks."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Sq, D = q.shape
    Sk = k.shape[0]
    if block <= 0:
        raise ValueError("block must be positive")
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((Sq, v.shape[1]))
    lse = np.zeros(Sq)
    for i in range(Sq):
        m = -np.inf
        d = 0.0
        acc = np.zeros(v.shape[1])
        for j0 in range(0, Sk, block):
            j1 = min(Sk, j0 + block)
            s = scale * (k[j0:j1] @ q[i])
            if causal:
                s = np.where(np.arange(j0, j1) > i, -np.inf, s)
            blk_max = s.max()
            if blk_max == -np.inf:
                continue  # a fully masked block changes nothing
            m_new = max(m, blk_max)
            corr = np.exp(m - m_new)  # exp(-inf) = 0 on the first block
            p = np.exp(s - m_new)
            d = d * corr + p.sum()
            acc = acc * corr + p @ v[j0:j1]
            m = m_new
        out[i] = acc / d
        lse[i] = m + np.log(d)
    return out, lse
