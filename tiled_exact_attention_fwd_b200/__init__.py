"""Python binding of libfa (include/fa.h): exact attention forward on B200 (sm_100a).

This module only marshals torch CUDA tensors into the C ABI: every step of the
computation runs in the library's kernels. There is no fallback: if libfa.so is not
built, every call raises.

    out, lse = fa_fwd(q, k, v, causal=True)                         # dense (B, S, H, D)
    out, lse = fa_varlen_fwd(q, k, v, cu_seqlens, max_seqlen)        # packed (total, H, D)
    out, lse = fa_fwd_paged(q, k_cache, v_cache, block_table)        # K/V in a page pool
    dq, dk, dv = fa_bwd(q, k, v, out, dout, lse, causal=True)        # gradients (recomputation)
    x_unpad  = fa_unpad(x, indices)                                  # (B, L, H, D) -> (nnz, H, D)
    x_pad    = fa_pad(x_unpad, indices, batch, total_len)            # (nnz, H, D) -> (B, L, H, D)
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_OK = 0
FA_FP16 = 0
FA_BF16 = 1
STATUS = {0: "FA_OK", -1: "FA_ERR_NULL", -2: "FA_ERR_SHAPE", -3: "FA_ERR_DTYPE", -4: "FA_ERR_HEADDIM",
          -5: "FA_ERR_ALIGN", -6: "FA_ERR_CUDA", -7: "FA_ERR_TIMEOUT", -8: "FA_ERR_INDEX"}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().fa_status_string(status).decode()} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m tiled_exact_attention_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, i32, vp]
        L.fa_varlen_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, i32, i32, f32, i32, i32, vp]
        L.fa_fwd_paged.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, i32, i32, i32, i32, f32, i32, i32, vp]
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, i32, vp]
        L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, i32, i32, vp]
        L.fa_varlen_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, vp, i32, i32, f32, i32, i32,
                                    vp]
        L.fa_unpad.argtypes = [vp, vp, i64, i64, i64, vp, vp]
        L.fa_pad.argtypes = [vp, vp, i64, i64, i64, vp, vp]
        L.fa_unpad_qkv.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp]
        L.fa_varlen_fwd_padded.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i64, vp, vp, i32, i32, f32, i32, i32,
                                           vp]
        L.fa_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), vp]
        L.fa_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp]
        for f in (L.fa_fwd, L.fa_fwd_paged, L.fa_bwd, L.fa_bwd_noalloc, L.fa_varlen_bwd, L.fa_varlen_fwd, L.fa_varlen_fwd_padded, L.fa_unpad, L.fa_unpad_qkv, L.fa_pad,
                  L.fa_device_status,
                  L.fa_selftest_bounded_wait):
            f.restype = ctypes.c_int
        L.fa_status_string.argtypes = [ctypes.c_int]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_version.argtypes = []
        L.fa_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != FA_OK:
        raise FAError(status, what)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float16 or bfloat16")


def _cuda_contig(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _shape(name: str, t: torch.Tensor, shape, dtype) -> None:
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _like(name: str, t: torch.Tensor, shape, dtype) -> None:
    """A caller-given output or workspace: exactly `shape` and `dtype` (the library writes every
    element of that shape, so a smaller buffer would be overrun), CUDA and contiguous."""
    _shape(name, t, shape, dtype)
    _cuda_contig(name, t)


def _on_device(t: torch.Tensor):
    """The operands' device made current for the call (a no-op context when it already is, which
    keeps the per-call host cost of small problems down)."""
    if t.get_device() == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(t.device)


def _same_device(ref: torch.Tensor, *ts: Optional[torch.Tensor]) -> None:
    for t in ts:
        if t is not None and t.device != ref.device:
            raise ValueError(f"every tensor must be on {ref.device}; got one on {t.device}")


def fa_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[torch.Tensor] = None,
           lse: Optional[torch.Tensor] = None, scale: Optional[float] = None, causal: bool = False,
           return_lse: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Dense forward: q, k, v (B, S, H, D) -> out (B, S, H, D), lse (B, H, S) fp32."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda_contig(n, t)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one (B, S, H, D) shape and dtype")
    B, S, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _like("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty((B, H, S), device=q.device, dtype=torch.float32)
    if lse is not None:
        _like("lse", lse, (B, H, S), torch.float32)
    _same_device(q, k, v, out, lse)
    with _on_device(q):
        st = lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, S, D,
                          float(scale) if scale else 0.0, int(bool(causal)), _dtype_code(q), _stream(stream))
    _check(st, "fa_fwd")
    return out, lse


def fa_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
           lse: torch.Tensor, dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
           dv: Optional[torch.Tensor] = None, delta: Optional[torch.Tensor] = None, scale: Optional[float] = None,
           causal: bool = False, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Dense backward: gradients (dq, dk, dv), each (B, S, H, D), of out = fa_fwd(q, k, v) given
    dout and the forward's lse (B, H, S). `delta` is an optional fp32 (B, H, S) workspace."""
    if q.dim() != 4 or any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, out, dout)):
        raise ValueError("q, k, v, out, dout must share one (B, S, H, D) shape and dtype")
    B, S, H, D = q.shape
    _shape("lse", lse, (B, H, S), torch.float32)
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if t is not None:
            _shape(n, t, q.shape, q.dtype)
    if delta is not None:
        _shape("delta", delta, (B, H, S), torch.float32)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse)):
        _cuda_contig(n, t)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if delta is None:
        delta = torch.empty((B, H, S), device=q.device, dtype=torch.float32)
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _like(n, t, q.shape, q.dtype)
    _like("delta", delta, (B, H, S), torch.float32)
    _same_device(q, k, v, out, dout, lse, dq, dk, dv, delta)
    with _on_device(q):
        st = lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                          _ptr(dv), _ptr(delta), B, H, S, D, float(scale) if scale else 0.0, int(bool(causal)),
                          _dtype_code(q), _stream(stream))
    _check(st, "fa_bwd")
    return dq, dk, dv


def fa_varlen_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                  lse: torch.Tensor, cu_seqlens: torch.Tensor, max_seqlen: int, scale: Optional[float] = None,
                  causal: bool = False, stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Packed backward: (total, H, D) tensors, lse (H, total) from fa_varlen_fwd -> (dq, dk, dv)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse),
                 ("cu_seqlens", cu_seqlens)):
        _cuda_contig(n, t)
    if q.dim() != 3 or any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, out, dout)):
        raise ValueError("q, k, v, out, dout must share one (total, H, D) shape and dtype")
    total, H, D = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (H, total):
        raise ValueError("lse must be float32 (H, total)")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    delta = torch.empty((H, total), device=q.device, dtype=torch.float32)
    _same_device(q, k, v, out, dout, lse, cu_seqlens)
    with _on_device(q):
        st = lib().fa_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(cu_seqlens),
                                 cu_seqlens.numel() - 1, int(max_seqlen), total, _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(delta), H, D, float(scale) if scale else 0.0, int(bool(causal)), _dtype_code(q),
                                 _stream(stream))
    _check(st, "fa_varlen_bwd")
    return dq, dk, dv


def fa_bwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                   lse: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor,
                   scale: Optional[float] = None, causal: bool = False, stream=None) -> None:
    """fa_bwd into caller-given dq, dk, dv with the library's fixed delta buffer (no
    allocation by the library; concurrent calls share that buffer and must be serialised).
    Every tensor is checked here, because the library takes B, H, S, D from q alone."""
    if q.dim() != 4 or any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, out, dout)):
        raise ValueError("q, k, v, out, dout must share one (B, S, H, D) shape and dtype")
    B, S, H, D = q.shape
    _shape("lse", lse, (B, H, S), torch.float32)
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _shape(n, t, q.shape, q.dtype)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse), ("dq", dq),
                 ("dk", dk), ("dv", dv)):
        _cuda_contig(n, t)
    _same_device(q, k, v, out, dout, lse, dq, dk, dv)
    # the fixed buffer is looked up on the current device: make it q's
    with _on_device(q):
        st = lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq),
                                  _ptr(dk), _ptr(dv), B, H, S, D, float(scale) if scale else 0.0, int(bool(causal)),
                                  _dtype_code(q), _stream(stream))
    _check(st, "fa_bwd_noalloc")


def attention_bwd_flops(B: int, H: int, S: int, D: int, causal: bool) -> float:
    """Backward FLOPs by the usual convention: 2.5x the forward (five S x S x D products)."""
    return 2.5 * attention_flops(B, H, S, S, D, causal)


def fa_fwd_paged(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 scale: Optional[float] = None, causal: bool = False, return_lse: bool = True,
                 stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Dense forward with paged K/V: q (B, S, H, D); k_cache, v_cache (num_pages, page_size, H, D);
    block_table int32 (B, max_blocks_per_seq) -> out (B, S, H, D), lse (B, H, S) fp32."""
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("block_table", block_table)):
        _cuda_contig(n, t)
    if q.dim() != 4 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("q must be (B, S, H, D) and k_cache, v_cache one (num_pages, page_size, H, D) shape")
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("q, k_cache, v_cache must share one dtype")
    B, S, H, D = q.shape
    num_pages, page_size = k_cache.shape[0], k_cache.shape[1]
    if tuple(k_cache.shape[2:]) != (H, D):
        raise ValueError("k_cache and v_cache pages must hold (H, D) rows like q")
    if block_table.dtype != torch.int32 or block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be an int32 (B, max_blocks_per_seq) tensor")
    if out is None:
        out = torch.empty_like(q)
    _like("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty((B, H, S), device=q.device, dtype=torch.float32)
    if lse is not None:
        _like("lse", lse, (B, H, S), torch.float32)
    _same_device(q, k_cache, v_cache, block_table, out, lse)
    with _on_device(q):
        st = lib().fa_fwd_paged(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
                                page_size, num_pages, _ptr(out), _ptr(lse), B, H, S, D,
                                float(scale) if scale else 0.0, int(bool(causal)), _dtype_code(q), _stream(stream))
    _check(st, "fa_fwd_paged")
    return out, lse


def fa_varlen_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                  max_seqlen: int, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  scale: Optional[float] = None, causal: bool = False, return_lse: bool = True,
                  stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Packed forward: q, k, v (total, H, D) with int32 cu_seqlens -> out (total, H, D), lse (H, total)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens)):
        _cuda_contig(n, t)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one (total, H, D) shape and dtype")
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor")
    total, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _like("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty((H, total), device=q.device, dtype=torch.float32)
    if lse is not None:
        _like("lse", lse, (H, total), torch.float32)
    _same_device(q, k, v, cu_seqlens, out, lse)
    with _on_device(q):
        st = lib().fa_varlen_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), cu_seqlens.numel() - 1,
                                 int(max_seqlen), total, _ptr(out), _ptr(lse), H, D,
                                 float(scale) if scale else 0.0, int(bool(causal)), _dtype_code(q), _stream(stream))
    _check(st, "fa_varlen_fwd")
    return out, lse


def fa_varlen_fwd_padded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, indices: torch.Tensor,
                         cu_seqlens: torch.Tensor, max_seqlen: int, out: Optional[torch.Tensor] = None,
                         lse: Optional[torch.Tensor] = None, scale: Optional[float] = None, causal: bool = False,
                         return_lse: bool = True, stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Fused unpad -> packed attention -> pad: padded q, k, v (..., H, D) with the int64 padded row
    of every packed token -> padded out (zeros at padding rows), lse (H, total)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("indices", indices), ("cu_seqlens", cu_seqlens)):
        _cuda_contig(n, t)
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one shape and dtype")
    if indices.dtype != torch.int64 or cu_seqlens.dtype != torch.int32:
        raise ValueError("indices must be int64 and cu_seqlens int32")
    H, D = q.shape[-2], q.shape[-1]
    padded_rows = q.numel() // (H * D)
    total = indices.numel()
    if out is None:
        out = torch.empty_like(q)
    _like("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty((H, total), device=q.device, dtype=torch.float32)
    if lse is not None:
        _like("lse", lse, (H, total), torch.float32)
    _same_device(q, k, v, indices, cu_seqlens, out, lse)
    with _on_device(q):
        st = lib().fa_varlen_fwd_padded(_ptr(q), _ptr(k), _ptr(v), _ptr(indices), _ptr(cu_seqlens),
                                        cu_seqlens.numel() - 1, int(max_seqlen), total, padded_rows, _ptr(out),
                                        _ptr(lse), H, D, float(scale) if scale else 0.0, int(bool(causal)),
                                        _dtype_code(q), _stream(stream))
    _check(st, "fa_varlen_fwd_padded")
    return out, lse


def fa_unpad(x: torch.Tensor, indices: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """(B, L, H, D) (or any (..., H, D)) -> (nnz, H, D): rows taken by int64 indices."""
    _cuda_contig("x", x)
    _cuda_contig("indices", indices)
    if indices.dtype != torch.int64:
        raise ValueError("indices must be int64")
    H, D = x.shape[-2], x.shape[-1]
    row_bytes = H * D * x.element_size()
    total_rows = x.numel() // (H * D)
    nnz = indices.numel()
    if out is None:
        out = torch.empty((nnz, H, D), device=x.device, dtype=x.dtype)
    _like("out", out, (nnz, H, D), x.dtype)
    _same_device(x, indices, out)
    with _on_device(x):
        st = lib().fa_unpad(_ptr(x), _ptr(indices), nnz, total_rows, row_bytes, _ptr(out), _stream(stream))
    _check(st, "fa_unpad")
    return out


def fa_unpad_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, indices: torch.Tensor, outs=None,
                 stream=None):
    """The three gathers of the packed path in one launch: returns (q_unpad, k_unpad, v_unpad)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("indices", indices)):
        _cuda_contig(n, t)
    if k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one shape and dtype")
    if indices.dtype != torch.int64:
        raise ValueError("indices must be int64")
    H, D = q.shape[-2], q.shape[-1]
    nnz = indices.numel()
    if outs is None:
        outs = tuple(torch.empty((nnz, H, D), device=q.device, dtype=q.dtype) for _ in range(3))
    for i, o in enumerate(outs):
        _like(f"outs[{i}]", o, (nnz, H, D), q.dtype)
    _same_device(q, k, v, indices, *outs)
    with _on_device(q):
        st = lib().fa_unpad_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(indices), nnz, q.numel() // (H * D),
                                H * D * q.element_size(), _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                _stream(stream))
    _check(st, "fa_unpad_qkv")
    return outs


def fa_pad(x: torch.Tensor, indices: torch.Tensor, batch: int, total_len: int,
           out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """(nnz, H, D) -> (batch, total_len, H, D): rows put back by int64 indices, zeros elsewhere."""
    _cuda_contig("x", x)
    _cuda_contig("indices", indices)
    if indices.dtype != torch.int64:
        raise ValueError("indices must be int64")
    nnz, H, D = x.shape
    if indices.numel() != nnz:
        raise ValueError("indices must hold one entry per row of x")
    if out is None:
        out = torch.empty((batch, total_len, H, D), device=x.device, dtype=x.dtype)
    _like("out", out, (batch, total_len, H, D), x.dtype)
    _same_device(x, indices, out)
    with _on_device(x):
        st = lib().fa_pad(_ptr(x), _ptr(indices), nnz, batch * total_len, H * D * x.element_size(), _ptr(out),
                          _stream(stream))
    _check(st, "fa_pad")
    return out


def fa_device_status(stream=None, device=None) -> Tuple[int, int]:
    """(status, where) recorded by kernels on the device since the last call. Waits for `stream`
    only (default: the current stream of `device`, default the current device)."""
    where = ctypes.c_int(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if isinstance(stream, torch.cuda.Stream):
        dev = stream.device
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev).cuda_stream if stream is None else _stream(stream)
        st = lib().fa_device_status(ctypes.byref(where), s)
    return st, where.value


def fa_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(lib().fa_selftest_bounded_wait(int(limit_ns), _stream(stream)), "fa_selftest_bounded_wait")


def version() -> str:
    return lib().fa_version().decode()


def attention_flops(B: int, H: int, Sq: int, Sk: int, D: int, causal: bool) -> float:
    """4*B*H*Sq*Sk*D (two matmuls of 2*Sq*Sk*D each), halved for causal."""
    f = 4.0 * B * H * Sq * Sk * D
    return f / 2 if causal else f
