"""Float64 CPU oracle for the attention forward path.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg are the only callers. The product library never imports this package,
and this package imports nothing from the product library; the two share only the seeded
input generators of ``fa_inputs``.

The arithmetic lives in ``fa_oracle.c`` (plain loops, float64, OpenMP over query rows);
this module marshals torch/numpy arrays into it. ``online_softmax.py`` holds the pages'
blockwise online-softmax merge, used only to check the claim that it reproduces the
full softmax.

Each function's docstring cites the passage it follows. Where the pages are silent the
reading taken is stated (scale default 1/sqrt(D); natural-log LSE of scaled scores;
causal mask aligned per sequence; zero fill for pad).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libfa_oracle.so")
_lib = None

_i64p = ctypes.POINTER(ctypes.c_int64)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile ``fa_oracle.c`` with gcc (-O2, OpenMP, no fast-math) into ``libfa_oracle.so``."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.fa_oracle_max_threads.restype = ctypes.c_int
        L.fa_oracle_attention_rows.restype = ctypes.c_int
        L.fa_oracle_attention_rows.argtypes = [
            _f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            _i64p, _i64p, _i64p, _i64p, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
            _f64p, _f64p, _f64p, ctypes.c_int64, ctypes.c_int]
        for name in ("fa_oracle_unpad", "fa_oracle_pad"):
            f = getattr(L, name)
            f.restype = ctypes.c_int
            f.argtypes = [_u8p, _i64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _u8p]
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().fa_oracle_max_threads())


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def attention_rows(q, k, v, tok, head, lo, hi, scale: Optional[float] = None,
                   causal: bool = False, want_probs: bool = False, nthreads: int = 0):
    """Output rows and LSE of standard attention for chosen query rows.

    Standard attention as defined on page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下",
    section "传统实现到底慢在哪": scores = Q K^T * scale, softmax over the key window,
    multiplied by V; causal masking per section "昇腾NPU上做了什么特殊优化".

    q, k, v: token-major (N, H, D). Row r is query token ``tok[r]`` of head ``head[r]``
    attending to keys [lo[r], hi[r]). Returns (out (n, D), lse (n,), probs or None).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one (N, H, D) shape")
    N, H, D = q.shape
    tok, head, lo, hi = _i64(tok), _i64(head), _i64(lo), _i64(hi)
    n = int(tok.size)
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    win = int((hi - lo).max()) if n else 0
    probs = np.zeros((n, max(win, 1)), dtype=np.float64) if want_probs else None
    rc = lib().fa_oracle_attention_rows(
        _ptr(q, _f64p), _ptr(k, _f64p), _ptr(v, _f64p), N, H, D,
        _ptr(tok, _i64p), _ptr(head, _i64p), _ptr(lo, _i64p), _ptr(hi, _i64p), n,
        float(scale) if scale is not None else 0.0, int(bool(causal)),
        _ptr(out, _f64p), _ptr(lse, _f64p),
        _ptr(probs, _f64p) if probs is not None else None, max(win, 1), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (status {rc})")
    return out, lse, probs


def dense_row_spec(B: int, S: int, H: int, rows=None, causal: bool = False):
    """(tok, head, lo, hi) for rows (b, h, i) of a dense (B, S, H, D) problem (all if None)."""
    if rows is None:
        b, h, i = np.meshgrid(np.arange(B), np.arange(H), np.arange(S), indexing="ij")
        b, h, i = b.ravel(), h.ravel(), i.ravel()
    else:
        rows = _i64(rows).reshape(-1, 3)
        b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    return b * S + i, h, b * S, b * S + S


def attention_dense(q, k, v, scale: Optional[float] = None, causal: bool = False,
                    rows=None, nthreads: int = 0):
    """Dense (B, S, H, D) attention.

    rows None: returns (O (B, S, H, D), LSE (B, H, S)) float64 over every row.
    rows given as an (n, 3) array of (b, h, i): returns (O_rows (n, D), LSE_rows (n,)).
    """
    B, S, H, D = q.shape
    tok, head, lo, hi = dense_row_spec(B, S, H, rows, causal)
    flat = lambda t: t.reshape(B * S, H, D)
    out, lse, _ = attention_rows(flat(q), flat(k), flat(v), tok, head, lo, hi, scale, causal,
                                 nthreads=nthreads)
    if rows is not None:
        return out, lse
    # row order of dense_row_spec is (b, h, i)
    O = out.reshape(B, H, S, D).transpose(0, 2, 1, 3).copy()
    L = lse.reshape(B, H, S)
    return O, L


def paged_to_contiguous(cache: torch.Tensor, block_table, S: int) -> torch.Tensor:
    """Key positions 0..S-1 of every batch entry read out of a page pool: (B, S, H, D).

    Page mooersco.com "FlashAttention 的“加速玄学”", section 5, recommends PagedAttention
    without giving a layout; the block-table reading is: position pos of entry b is row
    pos % page_size of page block_table[b][pos // page_size] of the (num_pages, page_size,
    H, D) pool. A plain copy, page by page.
    """
    bt = _i64(block_table)
    B = bt.shape[0]
    page_size = cache.shape[1]
    out = torch.empty((B, S) + tuple(cache.shape[2:]), dtype=cache.dtype)
    for b in range(B):
        for lp in range((S + page_size - 1) // page_size):
            n = min(page_size, S - lp * page_size)
            out[b, lp * page_size:lp * page_size + n] = cache[int(bt[b, lp]), :n]
    return out


def attention_paged(q, k_cache, v_cache, block_table, scale: Optional[float] = None, causal: bool = False,
                    rows=None, nthreads: int = 0):
    """Dense attention of q (B, S, H, D) over K/V held in page pools: the dense definition
    applied to the keys and values the block table describes (``paged_to_contiguous``)."""
    S = q.shape[1]
    k = paged_to_contiguous(k_cache, block_table, S)
    v = paged_to_contiguous(v_cache, block_table, S)
    return attention_dense(q, k, v, scale=scale, causal=causal, rows=rows, nthreads=nthreads)


def varlen_row_spec(cu_seqlens, H: int, rows=None):
    """(tok, head, lo, hi) for packed rows; rows None = all, else an (n, 2) array of (token, head)."""
    cu = _i64(cu_seqlens)
    total = int(cu[-1])
    seq_of = np.zeros(total, dtype=np.int64)
    for s in range(len(cu) - 1):
        seq_of[cu[s]:cu[s + 1]] = s
    if rows is None:
        t, h = np.meshgrid(np.arange(total), np.arange(H), indexing="ij")
        t, h = t.ravel(), h.ravel()
    else:
        rows = _i64(rows).reshape(-1, 2)
        t, h = rows[:, 0], rows[:, 1]
    s = seq_of[t]
    return t, h, cu[s], cu[s + 1]


def attention_varlen(q, k, v, cu_seqlens, scale: Optional[float] = None, causal: bool = False,
                     rows=None, nthreads: int = 0):
    """Packed (total, H, D) attention, each sequence [cu[s], cu[s+1]) attending only to itself.

    The packed path of page "IAW 模型 FA2 vs FA3 实测", section 1 (flash_attn_varlen_func on
    the compact tensor). rows None: (O (total, H, D), LSE (H, total)); rows given as an
    (n, 2) array of (token, head): (O_rows (n, D), LSE_rows (n,)).
    """
    total, H, D = q.shape
    tok, head, lo, hi = varlen_row_spec(cu_seqlens, H, rows)
    keep = hi > lo
    out, lse, _ = attention_rows(q, k, v, tok[keep], head[keep], lo[keep], hi[keep], scale, causal,
                                 nthreads=nthreads)
    if rows is not None:
        return out, lse
    O = np.zeros((total, H, D))
    L = np.zeros((H, total))
    O[tok[keep], head[keep]] = out
    L[head[keep], tok[keep]] = lse
    return O, L


def _rows_u8(x: torch.Tensor, rows: int) -> np.ndarray:
    a = x.detach().cpu().contiguous().view(torch.uint8).numpy().reshape(rows, -1)
    return np.ascontiguousarray(a)


def unpad(x: torch.Tensor, indices) -> torch.Tensor:
    """Gather rows of a padded (B, total_len, H, D) tensor into (nnz, H, D).

    Page "IAW 模型 FA2 vs FA3 实测", section 1: unpad drops the padding tokens by taking
    rows by ``indices`` (a gather).
    """
    H, D = x.shape[-2], x.shape[-1]
    total_rows = x.numel() // (H * D)
    idx = _i64(indices)
    if idx.size == 0:
        return torch.zeros((0, H, D), dtype=x.dtype)
    xs = _rows_u8(x, total_rows)
    row_bytes = xs.shape[1] if total_rows else H * D * x.element_size()
    out = np.zeros((idx.size, row_bytes), dtype=np.uint8)
    rc = lib().fa_oracle_unpad(_ptr(xs, _u8p), _ptr(idx, _i64p), idx.size, total_rows, row_bytes,
                               _ptr(out, _u8p))
    if rc != 0:
        raise ValueError(f"oracle unpad rejected its arguments (status {rc})")
    return torch.from_numpy(out).view(x.dtype).reshape(idx.size, H, D)


def pad(x: torch.Tensor, indices, batch: int, total_len: int) -> torch.Tensor:
    """Scatter packed (nnz, H, D) rows back to (batch, total_len, H, D); other rows are zero.

    Page "IAW 模型 FA2 vs FA3 实测", section 1 (scatter by indices) and section 2 (pad is a
    zero fill followed by an index put).
    """
    nnz, H, D = x.shape
    row_bytes = H * D * x.element_size()
    xs = _rows_u8(x, nnz) if nnz else np.zeros((0, row_bytes), dtype=np.uint8)
    idx = _i64(indices)
    total_rows = batch * total_len
    out = np.zeros((total_rows, row_bytes), dtype=np.uint8)
    rc = lib().fa_oracle_pad(_ptr(xs, _u8p), _ptr(idx, _i64p), nnz, total_rows, row_bytes,
                             _ptr(out, _u8p))
    if rc != 0:
        raise ValueError(f"oracle pad rejected its arguments (status {rc})")
    return torch.from_numpy(out).view(x.dtype).reshape(batch, total_len, H, D)


from .online_softmax import online_softmax_attention  # noqa: E402,F401
from .backward import attention_backward, attention_backward_head, attention_varlen_backward  # noqa: E402,F401
