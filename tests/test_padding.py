"""unpad / pad on the GPU vs the oracle's byte loops: bit-exact (needs a B200)."""
import pytest
import torch

import fa_inputs
import oracle
import tiled_exact_attention_fwd_b200 as fa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    fa.lib()


def _bits(t):
    return t.contiguous().view(torch.uint8)


@pytest.mark.parametrize("shape", [(1, 4096, 16, 128), (3, 100, 3, 8), (2, 37, 1, 7), (1, 1000, 4, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0, 0.03])
def test_unpad_pad_bit_exact(shape, dtype, frac):
    B, L, H, D = shape
    total = B * L
    nnz = int(round(total * frac))
    x = fa_inputs.normal(shape, dtype, seed=total + nnz)
    idx = fa_inputs.valid_indices(total, nnz, seed=nnz + 1)
    dev = torch.device("cuda:0")
    u = fa.fa_unpad(x.to(dev), idx.to(dev))
    torch.cuda.synchronize()
    u_ref = oracle.unpad(x, idx)
    assert torch.equal(_bits(u.cpu()), _bits(u_ref))
    p = fa.fa_pad(u, idx.to(dev), B, L)
    torch.cuda.synchronize()
    p_ref = oracle.pad(u_ref, idx, B, L)
    assert torch.equal(_bits(p.cpu()), _bits(p_ref))


def test_pad_overwrites_every_row():
    """Output rows no index names must become zero even if the buffer held garbage."""
    dev = torch.device("cuda:0")
    x = fa_inputs.normal((50, 2, 16), torch.bfloat16, 3).to(dev)
    idx = fa_inputs.valid_indices(200, 50, 4).to(dev)
    out = torch.full((1, 200, 2, 16), float("nan"), dtype=torch.bfloat16, device=dev)
    fa.fa_pad(x, idx, 1, 200, out=out)
    ref = oracle.pad(x.cpu(), idx.cpu(), 1, 200)
    assert torch.equal(_bits(out.cpu()), _bits(ref))


def test_unaligned_row_bytes_use_byte_path():
    dev = torch.device("cuda:0")
    x = torch.arange(5 * 9 * 1 * 3, dtype=torch.uint8).reshape(1, 45, 1, 3)  # 3-byte rows
    idx = torch.tensor([0, 4, 5, 44], dtype=torch.int64)
    u = fa.fa_unpad(x.to(dev), idx.to(dev)).cpu()
    assert torch.equal(u, oracle.unpad(x, idx))
    p = fa.fa_pad(u.to(dev), idx.to(dev), 1, 45).cpu()
    assert torch.equal(p, oracle.pad(u, idx, 1, 45))


@pytest.mark.parametrize("shape", [(1, 4096, 16, 128), (2, 50, 3, 8), (1, 33, 1, 7)])
def test_unpad_qkv_one_launch_bit_exact(shape):
    B, L, H, D = shape
    total = B * L
    nnz = total // 2 + 1
    q, k, v = (fa_inputs.normal(shape, torch.bfloat16, seed=s) for s in (1, 2, 3))
    idx = fa_inputs.valid_indices(total, nnz, seed=9)
    dev = torch.device("cuda:0")
    outs = fa.fa_unpad_qkv(q.to(dev), k.to(dev), v.to(dev), idx.to(dev))
    torch.cuda.synchronize()
    for x, o in zip((q, k, v), outs):
        assert torch.equal(_bits(o.cpu()), _bits(oracle.unpad(x, idx)))
