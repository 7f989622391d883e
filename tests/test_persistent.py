"""The dense forward's persistent grid (one CTA per SM running several work items) against the
float64 oracle, on shapes chosen to stress it (needs a B200): many more items than SMs, items
whose second query tile is absent (an odd number of 128-row tiles) mixed with full ones in the
same CTA, every head dim, causal and not, paged K/V, an output buffer that is 16- but not
32-byte aligned (the epilogue's narrower store path), and causal problems large enough that
the items are dealt in groups of heads."""
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


@pytest.mark.parametrize("B,H", [(1, 36), (2, 18)])
def test_head_groups_match_single_heads(B, H):
    """Causal S8192 D128 with 36 (batch entry, head) pairs: their K/V (144 MB) exceeds what the
    kernel keeps in L2, so the items are dealt in groups of heads (8, 8, 8, 8 and a partial 4,
    crossing batch entries when B = 2). Each pair's output and LSE must equal, bit for bit, those
    of a call on that pair alone (one group); rows of one pair are checked against the oracle."""
    S, D, dtype = 8192, 128, torch.bfloat16
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in fa_inputs.dense_qkv(B, S, H, D, dtype, seed=5))
    out, lse = fa.fa_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    for bh in [0, 7, 8, 15, 16, 31, 32, 35]:
        b, h = divmod(bh, H)
        qs, ks, vs = (t[b:b + 1, :, h:h + 1].contiguous() for t in (q, k, v))
        o1, l1 = fa.fa_fwd(qs, ks, vs, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(out[b:b + 1, :, h:h + 1], o1), f"output of pair {bh}"
        assert torch.equal(lse[b:b + 1, h:h + 1], l1), f"LSE of pair {bh}"
    # one pair's rows against the oracle (that head alone, float64 on the CPU)
    b, h = divmod(33, H)
    qh, kh, vh = (t[b:b + 1, :, h:h + 1].cpu() for t in (q, k, v))
    idx = np.array([0, 1, 127, 128, 4095, 8000, 8191])
    rows = np.stack([np.zeros_like(idx), np.zeros_like(idx), idx], axis=1)
    O, L = oracle.attention_dense(qh, kh, vh, causal=True, rows=rows)
    assert_o_close(out[b, idx, h].cpu(), O, dtype, "sampled rows")
    assert_lse_close(lse[b, h, idx].cpu(), L, "sampled rows")


def test_item_queue_repeated_calls_on_two_streams():
    """Non-causal B2 H40 S1024 D64 (320 items over the SMs) takes its items from the device item
    queue. 70 calls in a row (more than the 64 counter slots, so every slot is reused after the
    last CTA of its launch zeroed it), alternating between two streams without waiting, each
    into a NaN-filled output: every output and LSE must equal, bit for bit, those of the first
    call, and each (batch entry, head) those of a call on that pair alone (4 items, the static
    rounds); one pair is checked against the oracle."""
    B, S, H, D, dtype = 2, 1024, 40, 64, torch.bfloat16
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in fa_inputs.dense_qkv(B, S, H, D, dtype, seed=21))
    ref, ref_lse = fa.fa_fwd(q, k, v)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    outs = []
    for i in range(70):
        s = streams[i % 2]
        with torch.cuda.stream(s):
            o = torch.full_like(q, float("nan"))
            l = torch.full((B, H, S), float("nan"), device=dev)
            fa.fa_fwd(q, k, v, out=o, lse=l, stream=s)
        outs.append((o, l))
    torch.cuda.synchronize()
    for i, (o, l) in enumerate(outs):
        assert torch.equal(o, ref), f"output of call {i}"
        assert torch.equal(l, ref_lse), f"LSE of call {i}"
    for b, h in [(0, 0), (0, 39), (1, 17)]:
        qs, ks, vs = (t[b:b + 1, :, h:h + 1].contiguous() for t in (q, k, v))
        o1, l1 = fa.fa_fwd(qs, ks, vs)
        torch.cuda.synchronize()
        assert torch.equal(ref[b:b + 1, :, h:h + 1], o1), f"output of pair ({b}, {h})"
        assert torch.equal(ref_lse[b:b + 1, h:h + 1], l1), f"LSE of pair ({b}, {h})"
    qh, kh, vh = (t[1:2, :, 17:18].cpu() for t in (q, k, v))
    O, L = oracle.attention_dense(qh, kh, vh, causal=False)
    assert_o_close(ref[1:2, :, 17:18].cpu(), O, dtype, "pair (1, 17)")
    assert_lse_close(ref_lse[1:2, 17:18].cpu(), L, "pair (1, 17)")


@pytest.mark.parametrize("D", [64, 256])
@pytest.mark.parametrize("extra", [1, 0])
@pytest.mark.parametrize("causal", [False, True])
def test_item_queue_round_boundaries(D, extra, causal):
    """Items = units + 1 (one unit takes a second item from the queue) and exactly twice the
    units (every unit takes one more), a unit being a CTA (D = 64) or a 2-CTA cluster (D = 256,
    whose CTA 0 takes the items for both): S256 has one item per (batch entry, head), so H
    sets the item count. Each head must equal, bit for bit, a call on that head alone (one
    item, no queue); two heads are checked against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    units = sms // 2 if D == 256 else sms
    H = units + 1 if extra else 2 * units
    B, S, dtype = 1, 256, torch.float16
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in fa_inputs.dense_qkv(B, S, H, D, dtype, seed=31 + extra))
    out, lse = fa.fa_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert not torch.isnan(out).any()
    for h in [0, 1, units - 1, units, H - 1]:
        qs, ks, vs = (t[:, :, h:h + 1].contiguous() for t in (q, k, v))
        o1, l1 = fa.fa_fwd(qs, ks, vs, causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(out[:, :, h:h + 1], o1), f"output of head {h}"
        assert torch.equal(lse[:, h:h + 1], l1), f"LSE of head {h}"
    for h in [0, H - 1]:
        qh, kh, vh = (t[:, :, h:h + 1].cpu() for t in (q, k, v))
        O, L = oracle.attention_dense(qh, kh, vh, causal=causal)
        assert_o_close(out[:, :, h:h + 1].cpu(), O, dtype, f"head {h}")
        assert_lse_close(lse[:, h:h + 1].cpu(), L, f"head {h}")
