"""Float64 gradients of standard attention: the oracle of the backward pass.

TEST INFRASTRUCTURE ONLY (see the package docstring): the test suite and the benchmark's
CPU-baseline leg are the only callers; nothing here is shared with the CUDA path.

Page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下", section "分块计算，这事没那么简单",
second pitfall ("反向传播怎么办"): the intermediate scores are not stored, the backward pass
recomputes the forward. The pages print no gradient formulas; the oracle is the plain
derivative of O = softmax(Z) V with Z = scale * Q K^T (masked scores weigh exactly 0),
written out per (batch, head) with full S x S matrices:

    P  = softmax(Z) row-wise
    dV = P^T dO
    dP = dO V^T
    dZ = P * (dP - rowsum(P * dP))
    dQ = scale * dZ K
    dK = scale * dZ^T Q
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def attention_backward_head(q, k, v, do, scale: Optional[float] = None, causal: bool = False):
    """Gradients (dq, dk, dv) of one head: q, k, v, do are (S, D); causal masks key j > query i."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    S, D = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    z = scale * (q @ k.T)
    if causal:
        z = np.where(np.triu(np.ones((S, S), dtype=bool), 1), -np.inf, z)
    z_max = z.max(axis=1, keepdims=True)
    w = np.exp(z - z_max)
    p = w / w.sum(axis=1, keepdims=True)
    dv = p.T @ do
    dp = do @ v.T
    dz = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    dq = scale * (dz @ k)
    dk = scale * (dz.T @ q)
    return dq, dk, dv


def attention_backward(q, k, v, dout, scale: Optional[float] = None, causal: bool = False, heads=None):
    """Gradients of dense (B, S, H, D) attention.

    heads None: (dq, dk, dv) float64 arrays (B, S, H, D) over every head.
    heads given as a list of (b, h): a dict {(b, h): (dq, dk, dv)} of (S, D) arrays.
    """
    B, S, H, D = q.shape
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else [tuple(x) for x in heads]
    res = {}
    for b, h in pairs:
        res[(b, h)] = attention_backward_head(q[b, :, h], k[b, :, h], v[b, :, h], dout[b, :, h], scale, causal)
    if heads is not None:
        return res
    dq = np.zeros((B, S, H, D))
    dk = np.zeros((B, S, H, D))
    dv = np.zeros((B, S, H, D))
    for (b, h), (gq, gk, gv) in res.items():
        dq[b, :, h], dk[b, :, h], dv[b, :, h] = gq, gk, gv
    return dq, dk, dv


def attention_varlen_backward(q, k, v, dout, cu_seqlens, scale: Optional[float] = None, causal: bool = False):
    """Gradients of packed (total, H, D) attention: each sequence [cu[s], cu[s+1]) on its own
    (page "IAW 模型 FA2 vs FA3 实测", section 1: the packed batch is attention within each
    sequence), by attention_backward_head per (sequence, head). Returns float64 (total, H, D)."""
    cu = [int(x) for x in (cu_seqlens.tolist() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens)]
    total, H, D = q.shape
    dq = np.zeros((total, H, D))
    dk = np.zeros((total, H, D))
    dv = np.zeros((total, H, D))
    for s0, s1 in zip(cu[:-1], cu[1:]):
        if s1 <= s0:
            continue
        for h in range(H):
            gq, gk, gv = attention_backward_head(q[s0:s1, h], k[s0:s1, h], v[s0:s1, h], dout[s0:s1, h], scale, causal)
            dq[s0:s1, h], dk[s0:s1, h], dv[s0:s1, h] = gq, gk, gv
    return dq, dk, dv
