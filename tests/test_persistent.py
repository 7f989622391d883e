"""The dense forward's persistent grid (one CTA per SM running several work items) against the
float64 oracle, on shapes chosen to stress it (needs a B200): many more items than SMs, items
whose second query tile is absent (an odd number of 128-row tiles) mixed with full ones in the
same CTA, every head dim, causal and not, paged K/V, and an output buffer that is 16- but not
32-byte aligned (the epilogue's narrower store path)."""
import numpy as np
import pytest
import torch

import fa_inputs
import oracle
import tiled_exact_attention_fwd_b200 as fa
from parity_util import assert_lse_close, assert_o_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    fa.lib()
    yield
    st, where = fa.fa_device_status()
    assert st == 0, f"device status {st} at {where}"


@pytest.mark.parametrize("D,H", [(64, 60), (128, 60), (256, 40)])
@pytest.mark.parametrize("causal", [False, True])
def test_many_items_per_cta(D, H, causal):
    """B2 S640 (five query tiles: the third item of every (batch, head) has no tile B): 360 or 400
    work items over the SMs, so each CTA runs two or three items of different kinds."""
    B, S, dtype = 2, 640, torch.bfloat16
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, dtype, seed=D + int(causal))
    dev = torch.device("cuda:0")
    out, lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal)
    torch.cuda.synchronize()
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    assert_o_close(out.cpu(), O, dtype, f"D={D} causal={causal}")
    assert_lse_close(lse.cpu(), L, f"D={D} causal={causal}")


@pytest.mark.parametrize("page_size", [16, 128])
def test_paged_many_items_matches_contiguous(page_size):
    """The paged kernel is persistent too: 3 x 50 heads x 3 items over the SMs, bit for bit
    equal to the contiguous forward on the keys the block table describes."""
    B, S, H, D, dtype = 3, 700, 50, 128, torch.bfloat16
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, dtype, seed=page_size)
    kc, vc, table = fa_inputs.paged_kv(k, v, page_size, seed=3, fill=float("nan"))
    dev = torch.device("cuda:0")
    ref, ref_lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    out, lse = fa.fa_fwd_paged(q.to(dev), kc.to(dev), vc.to(dev), table.to(dev), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    # and one batch entry's heads 0 and 49 against the oracle
    O, L = oracle.attention_dense(q[1:2, :, [0, 49]], k[1:2, :, [0, 49]], v[1:2, :, [0, 49]], causal=True)
    assert_o_close(out[1:2, :, [0, 49]].cpu(), O, dtype, "paged heads 0, 49")


@pytest.mark.parametrize("causal", [False, True])
def test_output_16_byte_aligned(causal):
    """out at a 16-byte (not 32-byte) boundary: the epilogue falls back to 16-byte stores and
    writes exactly the same values; nothing outside out is touched."""
    B, S, H, D, dtype = 1, 1000, 20, 64, torch.float16
    q, k, v = (t.cuda() for t in fa_inputs.dense_qkv(B, S, H, D, dtype, seed=5))
    ref, ref_lse = fa.fa_fwd(q, k, v, causal=causal)
    n = B * S * H * D
    buf = torch.full((n + 32,), 7.0, dtype=dtype, device="cuda")
    assert buf.data_ptr() % 32 == 0
    out = buf[8:8 + n].view(B, S, H, D)  # 16 bytes past a 32-byte boundary
    fa.fa_fwd(q, k, v, out=out, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert bool((buf[:8] == 7.0).all()) and bool((buf[8 + n:] == 7.0).all())
