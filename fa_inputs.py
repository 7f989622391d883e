"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module holds no attention arithmetic: it only draws random tensors, valid-token
masks and sequence boundaries, always on the CPU from a ``torch.Generator`` so that
the GPU path and the oracle see identical bits.

Workloads (shapes follow the pages' workloads; every value ~ N(0, 1)):

* ``dense_fp16_small``   B=1,  H=2,  S=128,  D=64,  fp16, non-causal
* ``varlen_bf16_32x64``  32 sequences x 64 tokens, H=16, D=128, bf16, padded (1, 4096, 16, 128)
                         with 2048 valid positions chosen at random
* ``vit_bf16``           B=149, H=12, S=1024, D=64, bf16, non-causal
* ``llm_causal_bf16``    B=1,  H=32, S=8192, D=128, bf16, causal
* ``hdim_sweep_fp16``    B=1,  S=4096, (H, D) in {(128,32),(64,64),(32,128),(16,256)}, fp16, causal

Sources for the shapes: "IAW 模型 FA2 vs FA3 实测" (section 1 packed path, section 5 table,
section 7 ViT table), "block_size和head_dim怎么选" (head_dim measurements at seq_len 4096),
"昇腾CANN跑大模型，FlashAttention这个算子你得认识一下" (13B model at sequence length 8192).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape: Sequence[int], dtype: torch.dtype, seed: int) -> torch.Tensor:
    """N(0,1) drawn in fp32 on the CPU, then rounded (RN) to ``dtype``."""
    return torch.randn(*shape, generator=generator(seed), dtype=torch.float32).to(dtype)


def dense_qkv(B: int, S: int, H: int, D: int, dtype: torch.dtype, seed: int = 0):
    """Contiguous (B, S, H, D) q, k, v on the CPU."""
    q = normal((B, S, H, D), dtype, seed * 3 + 0)
    k = normal((B, S, H, D), dtype, seed * 3 + 1)
    v = normal((B, S, H, D), dtype, seed * 3 + 2)
    return q, k, v


def cu_seqlens_from_lengths(lengths: Sequence[int]) -> torch.Tensor:
    """Running start offsets [0, l0, l0+l1, ...] as int32 (pure bookkeeping)."""
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def random_lengths(num_seqs: int, lo: int, hi: int, seed: int) -> List[int]:
    """Uniform integer sequence lengths in [lo, hi]."""
    g = generator(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (num_seqs,), generator=g)]


def valid_indices(total_len: int, nnz: int, seed: int) -> torch.Tensor:
    """Sorted flat positions of ``nnz`` valid tokens among ``total_len`` (int64).

    The positions are the first ``nnz`` entries of a seeded random permutation, sorted,
    which is what a nonzero() over a random 0/1 padding mask with ``nnz`` ones yields.
    """
    perm = torch.randperm(total_len, generator=generator(seed))
    return perm[:nnz].sort().values.to(torch.int64)


@dataclasses.dataclass
class VarlenCase:
    """A padded batch plus the bookkeeping that the packed path needs."""
    q_pad: torch.Tensor        # (1, total_len, H, D)
    k_pad: torch.Tensor
    v_pad: torch.Tensor
    indices: torch.Tensor      # int64 [nnz], sorted, unique
    cu_seqlens: torch.Tensor   # int32 [num_seqs + 1]
    max_seqlen: int
    H: int
    D: int

    @property
    def nnz(self) -> int:
        return int(self.indices.numel())

    @property
    def total_len(self) -> int:
        return int(self.q_pad.shape[1])


def varlen_case(lengths: Sequence[int], total_len: int, H: int, D: int,
                dtype: torch.dtype, seed: int = 0) -> VarlenCase:
    """Padded (1, total_len, H, D) q/k/v with sum(lengths) valid positions at random.

    The compact rows, taken in index order, form consecutive sequences of the given
    lengths (cu_seqlens), independent of where the valid positions fall.
    """
    nnz = int(sum(lengths))
    if nnz > total_len:
        raise ValueError("more valid tokens than positions")
    q, k, v = dense_qkv(1, total_len, H, D, dtype, seed)
    idx = valid_indices(total_len, nnz, seed + 7919)
    cu = cu_seqlens_from_lengths(lengths)
    return VarlenCase(q, k, v, idx, cu, int(max(lengths) if lengths else 0), H, D)


def right_padded_case(lengths: Sequence[int], slot: int, H: int, D: int,
                      dtype: torch.dtype, seed: int = 0) -> VarlenCase:
    """A (B, slot) batch with right padding, flattened to (1, B*slot, H, D): sequence b holds
    rows [b*slot, b*slot + lengths[b]), so its valid positions form one consecutive run."""
    if any(n > slot for n in lengths):
        raise ValueError("a sequence is longer than its slot")
    total_len = slot * len(lengths)
    q, k, v = dense_qkv(1, total_len, H, D, dtype, seed)
    idx = torch.tensor([b * slot + r for b, n in enumerate(lengths) for r in range(n)], dtype=torch.int64)
    cu = cu_seqlens_from_lengths(lengths)
    return VarlenCase(q, k, v, idx, cu, int(max(lengths) if lengths else 0), H, D)


def packed_qkv(lengths: Sequence[int], H: int, D: int, dtype: torch.dtype, seed: int = 0):
    """Packed (total, H, D) q, k, v plus int32 cu_seqlens, with no padding step."""
    total = int(sum(lengths))
    q = normal((total, H, D), dtype, seed * 3 + 0)
    k = normal((total, H, D), dtype, seed * 3 + 1)
    v = normal((total, H, D), dtype, seed * 3 + 2)
    return q, k, v, cu_seqlens_from_lengths(lengths)


# The five workloads. ``scale`` None means 1/sqrt(D).
WORKLOADS = {
    "dense_fp16_small": dict(kind="dense", B=1, H=2, S=128, D=64, dtype="fp16", causal=False),
    "varlen_bf16_32x64": dict(kind="varlen", lengths=[64] * 32, total_len=4096, H=16, D=128,
                              dtype="bf16", causal=False),
    "vit_bf16": dict(kind="dense", B=149, H=12, S=1024, D=64, dtype="bf16", causal=False),
    "llm_causal_bf16": dict(kind="dense", B=1, H=32, S=8192, D=128, dtype="bf16", causal=True),
    "hdim_sweep_fp16_d32": dict(kind="dense", B=1, H=128, S=4096, D=32, dtype="fp16", causal=True),
    "hdim_sweep_fp16_d64": dict(kind="dense", B=1, H=64, S=4096, D=64, dtype="fp16", causal=True),
    "hdim_sweep_fp16_d128": dict(kind="dense", B=1, H=32, S=4096, D=128, dtype="fp16", causal=True),
    "hdim_sweep_fp16_d256": dict(kind="dense", B=1, H=16, S=4096, D=256, dtype="fp16", causal=True),
}


def paged_kv(k: torch.Tensor, v: torch.Tensor, page_size: int, seed: int, spare_pages: int = 3,
             extra_table_cols: int = 1, fill: float = float("nan")):
    """Scatter contiguous (B, S, H, D) k and v into page pools of ``page_size`` rows.

    Pages are assigned in a seeded random order; ``spare_pages`` pages belong to no sequence.
    Rows of the pools that hold no key (spare pages, the tail of each sequence's last page)
    are set to ``fill``. The int32 block table has ``extra_table_cols`` more columns than a
    sequence needs, set to -1 (never read). Returns (k_cache, v_cache, block_table).
    """
    B, S, H, D = k.shape
    per_seq = (S + page_size - 1) // page_size
    num_pages = B * per_seq + spare_pages
    order = torch.randperm(num_pages, generator=generator(seed))
    table = torch.full((B, per_seq + extra_table_cols), -1, dtype=torch.int32)
    table[:, :per_seq] = order[:B * per_seq].reshape(B, per_seq).to(torch.int32)
    k_cache = torch.full((num_pages, page_size, H, D), fill, dtype=k.dtype)
    v_cache = torch.full((num_pages, page_size, H, D), fill, dtype=v.dtype)
    for b in range(B):
        for lp in range(per_seq):
            n = min(page_size, S - lp * page_size)
            pg = int(table[b, lp])
            k_cache[pg, :n] = k[b, lp * page_size:lp * page_size + n]
            v_cache[pg, :n] = v[b, lp * page_size:lp * page_size + n]
    return k_cache, v_cache, table


def workload_inputs(name: str, seed: int = 0):
    """CPU inputs of a named workload (dense: (q, k, v); varlen: VarlenCase)."""
    w = WORKLOADS[name]
    dt = DTYPES[w["dtype"]]
    if w["kind"] == "dense":
        return dense_qkv(w["B"], w["S"], w["H"], w["D"], dt, seed)
    return varlen_case(w["lengths"], w["total_len"], w["H"], w["D"], dt, seed)


def sample_rows(n_total: int, n: int, seed: int, must: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Sorted unique sample of ``n`` row ids out of ``n_total`` plus ``must`` (edge rows)."""
    g = generator(seed)
    pick = torch.randperm(n_total, generator=g)[: max(0, n)].tolist()
    if must:
        pick += [int(m) for m in must if 0 <= int(m) < n_total]
    return torch.tensor(sorted(set(pick)), dtype=torch.int64)
