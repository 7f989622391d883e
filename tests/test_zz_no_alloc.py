"""fa_bwd_noalloc: the backward pass with the library's fixed delta buffer instead of a
caller-owned workspace. Named to be collected last; it also passes on its own."""
import pytest
import torch

import fa_inputs

FAKE = 1 << 20  # a 16-byte aligned non-null address that is never dereferenced


def test_oversize_problem_is_refused_before_any_launch():
    import tiled_exact_attention_fwd_b200 as fa
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    L = fa.lib()
    # B * H * S = 2^24 + 128 rows > the 2^24-float buffer
    assert L.fa_bwd_noalloc(*([FAKE] * 9), 1, 128, 131073, 128, 0.0, 1, 1, None) == -2
    assert L.fa_bwd_noalloc(None, *([FAKE] * 8), 1, 1, 128, 128, 0.0, 1, 1, None) == -1
    assert L.fa_bwd_noalloc(*([FAKE] * 9), 1, 1, 128, 96, 0.0, 1, 1, None) == -4


@pytest.mark.gpu
@pytest.mark.parametrize("D", [128, 256])
def test_two_calls_match_the_workspace_entry_point(cuda_device, D):
    import tiled_exact_attention_fwd_b200 as fa
    dev = cuda_device
    for causal in (True, False):
        B, S, H = 2, 300, 4
        q, k, v = (t.to(dev) for t in fa_inputs.dense_qkv(B, S, H, D, torch.bfloat16, seed=9))
        do = fa_inputs.normal((B, S, H, D), torch.bfloat16, seed=10).to(dev)
        out, lse = fa.fa_fwd(q, k, v, causal=causal)
        ref = fa.fa_bwd(q, k, v, out, do, lse, causal=causal)
        for _ in range(2):  # two calls in a row on the same fixed buffer
            got = [torch.full_like(q, float("nan")) for _ in range(3)]
            fa.fa_bwd_noalloc(q, k, v, out, do, lse, *got, causal=causal)
            torch.cuda.synchronize()
            for g, r in zip(got, ref):
                assert torch.equal(g.view(torch.int16), r.view(torch.int16))
        assert fa.fa_device_status()[0] == 0
