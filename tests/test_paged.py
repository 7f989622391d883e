"""Paged K/V (the PagedAttention layout of page mooersco.com "FlashAttention 的“加速玄学”",
section 5; the block-table layout is this library's reading, the page gives none).

CPU: the oracle's page gather returns the contiguous keys exactly, whatever the pools hold
elsewhere. GPU: fa_fwd_paged against the oracle, and bit-for-bit against fa_fwd on the
contiguous tensors (same tiles, same arithmetic), with NaN in every pool row that holds no
key; an out-of-range page index is reported, not dereferenced.
"""
import pytest
import torch

import fa_inputs
import oracle
from parity_util import assert_o_close, assert_lse_close


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
def test_oracle_page_gather_is_exact(page_size):
    k, v, _ = fa_inputs.dense_qkv(3, 301, 2, 32, torch.bfloat16, seed=4)
    kc, vc, table = fa_inputs.paged_kv(k, v, page_size, seed=5)
    assert torch.isnan(kc.float()).any()  # the pools do hold NaN outside the keys
    for src, cache in ((k, kc), (v, vc)):
        got = oracle.paged_to_contiguous(cache, table, 301)
        assert torch.equal(got.view(torch.int16), src.view(torch.int16))


def test_oracle_paged_attention_is_dense_attention():
    q, k, v = fa_inputs.dense_qkv(2, 77, 2, 16, torch.float16, seed=6)
    kc, vc, table = fa_inputs.paged_kv(k, v, 16, seed=7)
    for causal in (False, True):
        O1, L1 = oracle.attention_paged(q, kc, vc, table, causal=causal)
        O2, L2 = oracle.attention_dense(q, k, v, causal=causal)
        assert (O1 == O2).all() and (L1 == L2).all()


CASES = [  # (D, page_size, dtype, causal)
    (32, 16, torch.bfloat16, True), (64, 64, torch.float16, False), (64, 16, torch.bfloat16, True),
    (128, 128, torch.bfloat16, True), (128, 32, torch.float16, False), (128, 256, torch.bfloat16, False),
    (128, 16, torch.bfloat16, True), (64, 32, torch.float16, True),
    (256, 64, torch.float16, True), (256, 128, torch.bfloat16, False), (256, 16, torch.bfloat16, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("D,page_size,dtype,causal", CASES)
def test_paged_matches_oracle_and_dense(cuda_device, D, page_size, dtype, causal):
    import tiled_exact_attention_fwd_b200 as fa
    B, S, H = 2, 333, 2  # 333: ragged last key tile and ragged last page
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, dtype, seed=D + page_size)
    kc, vc, table = fa_inputs.paged_kv(k, v, page_size, seed=11)
    dev = cuda_device
    out, lse = fa.fa_fwd_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), causal=causal)
    ref_out, ref_lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    assert_o_close(out.cpu(), O, dtype)
    assert_lse_close(lse.cpu(), L)


@pytest.mark.gpu
@pytest.mark.parametrize("page_size", [16, 64])
def test_paged_full_size_matches_dense(cuda_device, page_size):
    """The causal bf16 B1 H32 S8192 D128 workload in 16-row pages (copy producers) and 64-row
    pages (TMA), against fa_fwd on the contiguous tensors (bit for bit) and sampled rows of the
    oracle."""
    import tiled_exact_attention_fwd_b200 as fa
    B, S, H, D = 1, 8192, 32, 128
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, torch.bfloat16, seed=0)
    kc, vc, table = fa_inputs.paged_kv(k, v, page_size, seed=1, fill=0.0)
    dev = cuda_device
    out, lse = fa.fa_fwd_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), causal=True)
    ref_out, ref_lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    rows = torch.stack([torch.zeros(6, dtype=torch.long), torch.tensor([0, 5, 17, 31, 31, 9]),
                        torch.tensor([0, 1, 127, 4095, 8191, 6000])], dim=1)
    Or, Lr = oracle.attention_dense(q, k, v, causal=True, rows=rows.numpy())
    got = out.cpu()[0, rows[:, 2], rows[:, 1]]
    assert_o_close(got, Or, torch.bfloat16)
    assert_lse_close(lse.cpu()[0, rows[:, 1], rows[:, 2]], Lr)


@pytest.mark.gpu
def test_paged_bad_page_index_is_reported(cuda_device):
    import tiled_exact_attention_fwd_b200 as fa
    q, k, v = fa_inputs.dense_qkv(1, 200, 1, 64, torch.bfloat16, seed=2)
    kc, vc, table = fa_inputs.paged_kv(k, v, 64, seed=3, fill=0.0)
    table[0, 1] = kc.shape[0] + 5  # past the pool
    dev = cuda_device
    fa.fa_device_status()  # clear
    fa.fa_fwd_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev))
    torch.cuda.synchronize()
    code, _ = fa.fa_device_status()
    assert code == -8
    # the context is still usable
    out, _ = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
