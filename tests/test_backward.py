"""Backward pass (fa_bwd) against the float64 oracle of the attention derivative.

Tolerance: gradients are not O(1) (dK, dV of early keys sum over many queries), so the bar
is relative to each tensor's largest magnitude: max |gpu - oracle| <= tol * max(|oracle|, 0.01),
tol = 2e-2 for bf16 and 5e-3 for fp16 -- the forward's O tolerances, applied to the
normalised tensor. Error sources: P and dZ are rounded to the input type before the
P^T dO, dZ^T Q and dZ K products (relative 2^-9 bf16 / 2^-12 fp16 per element), delta is
computed from the rounded forward output, and the results are rounded once more.
"""
import numpy as np
import pytest
import torch

import fa_inputs
import oracle

TOL = {torch.bfloat16: 2e-2, torch.float16: 5e-3}


def _close(name, gpu, ref, dtype):
    g = gpu.detach().float().cpu().double().numpy()
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (name, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{name}: non-finite gradient"
    # a gradient that is exactly 0 in exact arithmetic (one key: dQ = dK = 0) comes out as
    # rounding noise; the floor keeps that case meaningful without loosening the others
    scale = max(float(np.abs(r).max()), 1e-2)
    err = float(np.abs(g - r).max()) / scale
    assert err <= TOL[dtype], f"{name}: max |gpu - oracle| / max |oracle| = {err:.3g} > {TOL[dtype]}"
    return err


def _run(B, S, H, D, dtype, causal, seed, dev):
    import tiled_exact_attention_fwd_b200 as fa
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, dtype, seed=seed)
    do = fa_inputs.normal((B, S, H, D), dtype, seed=seed + 100)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    out, lse = fa.fa_fwd(qd, kd, vd, causal=causal)
    dq, dk, dv = fa.fa_bwd(qd, kd, vd, out, dod, lse, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    return (q, k, v, do), (dq, dk, dv)


@pytest.mark.gpu
@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_oracle(cuda_device, D, dtype, causal):
    B, S, H = 2, 333, 2  # several tiles and a ragged last tile
    (q, k, v, do), (dq, dk, dv) = _run(B, S, H, D, dtype, causal, seed=D, dev=cuda_device)
    rq, rk, rv = oracle.attention_backward(q, k, v, do, causal=causal)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(name, g, r, dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("S", [1, 64, 128, 129])
def test_bwd_edge_lengths(cuda_device, S):
    """One key, a single partial tile, exactly one tile, one tile plus one row."""
    (q, k, v, do), (dq, dk, dv) = _run(1, S, 3, 64, torch.bfloat16, True, seed=S, dev=cuda_device)
    rq, rk, rv = oracle.attention_backward(q, k, v, do, causal=True)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(name, g, r, torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("S", [1, 64, 65, 129, 192])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_d256_edge_lengths(cuda_device, S, causal):
    """D = 256 streams 64-row half tiles: one key, exactly one half tile, one half tile plus one
    row, a tile plus one row, a tile and a half."""
    (q, k, v, do), (dq, dk, dv) = _run(1, S, 2, 256, torch.float16, causal, seed=S + 1, dev=cuda_device)
    rq, rk, rv = oracle.attention_backward(q, k, v, do, causal=causal)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(name, g, r, torch.float16)


@pytest.mark.gpu
def test_bwd_d256_long_causal_sampled_heads(cuda_device):
    """B1 H16 S2048 D256 causal bf16 (16 query tiles, 32 half-tile steps), two heads checked
    against the oracle over every row."""
    B, S, H, D = 1, 2048, 16, 256
    (q, k, v, do), (dq, dk, dv) = _run(B, S, H, D, torch.bfloat16, True, seed=11, dev=cuda_device)
    ref = oracle.attention_backward(q, k, v, do, causal=True, heads=[(0, 0), (0, 13)])
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            _close(f"{name}[h={h}]", g[b, :, h], r, torch.bfloat16)


@pytest.mark.gpu
def test_bwd_d256_long_noncausal_sampled_heads(cuda_device):
    """B1 H8 S1536 D256 non-causal fp16 (every key tile streams past every query tile), two
    heads checked against the oracle over every row."""
    B, S, H, D = 1, 1536, 8, 256
    (q, k, v, do), (dq, dk, dv) = _run(B, S, H, D, torch.float16, False, seed=13, dev=cuda_device)
    ref = oracle.attention_backward(q, k, v, do, causal=False, heads=[(0, 2), (0, 7)])
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            _close(f"{name}[h={h}]", g[b, :, h], r, torch.float16)


@pytest.mark.gpu
def test_bwd_long_causal_sampled_heads(cuda_device):
    """B1 H32 S4096 D128 causal bf16 (the head-dim sweep's D=128 shape), two heads checked
    against the oracle over every row."""
    B, S, H, D = 1, 4096, 32, 128
    (q, k, v, do), (dq, dk, dv) = _run(B, S, H, D, torch.bfloat16, True, seed=7, dev=cuda_device)
    ref = oracle.attention_backward(q, k, v, do, causal=True, heads=[(0, 0), (0, 21)])
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            _close(f"{name}[h={h}]", g[b, :, h], r, torch.bfloat16)


@pytest.mark.gpu
def test_bwd_delta_workspace_is_rowsum(cuda_device):
    """The caller's delta workspace holds rowsum(dout * out) in fp32 after the call."""
    import tiled_exact_attention_fwd_b200 as fa
    q, k, v = (t.to(cuda_device) for t in fa_inputs.dense_qkv(2, 200, 3, 64, torch.float16, seed=3))
    do = fa_inputs.normal((2, 200, 3, 64), torch.float16, seed=4).to(cuda_device)
    out, lse = fa.fa_fwd(q, k, v)
    delta = torch.full((2, 3, 200), float("nan"), device=cuda_device)
    fa.fa_bwd(q, k, v, out, do, lse, delta=delta)
    ref = (out.double() * do.double()).sum(-1).permute(0, 2, 1)
    torch.testing.assert_close(delta.double(), ref, rtol=1e-5, atol=1e-5)


@pytest.mark.gpu
@pytest.mark.parametrize("D,dtype,causal", [(64, torch.bfloat16, True), (128, torch.float16, False),
                                            (32, torch.bfloat16, False), (128, torch.bfloat16, True),
                                            (256, torch.bfloat16, True), (256, torch.float16, False)])
def test_varlen_bwd_matches_oracle(cuda_device, D, dtype, causal):
    """Packed sequences of mixed lengths (shorter than, equal to and longer than a tile, and
    empty), several sharing one 128-token tile."""
    import tiled_exact_attention_fwd_b200 as fa
    lengths = [5, 130, 0, 64, 1, 200, 63, 17]
    H = 2
    q, k, v, cu = fa_inputs.packed_qkv(lengths, H, D, dtype, seed=D)
    total = int(cu[-1])
    do = fa_inputs.normal((total, H, D), dtype, seed=D + 1)
    dev = cuda_device
    qd, kd, vd, dod, cud = (t.to(dev) for t in (q, k, v, do, cu))
    out, lse = fa.fa_varlen_fwd(qd, kd, vd, cud, max(lengths), causal=causal)
    dq, dk, dv = fa.fa_varlen_bwd(qd, kd, vd, out, dod, lse, cud, max(lengths), causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    rq, rk, rv = oracle.attention_varlen_backward(q, k, v, do, cu, causal=causal)
    for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        _close(name, g, r, dtype)


@pytest.mark.gpu
@pytest.mark.parametrize("D", [64, 256])
def test_varlen_bwd_single_sequence_equals_dense(cuda_device, D):
    """One packed sequence spanning everything gives exactly the dense kernels' gradients."""
    import tiled_exact_attention_fwd_b200 as fa
    S, H = 300, 2
    q, k, v = (t.to(cuda_device) for t in fa_inputs.dense_qkv(1, S, H, D, torch.bfloat16, seed=5))
    do = fa_inputs.normal((1, S, H, D), torch.bfloat16, seed=6).to(cuda_device)
    out, lse = fa.fa_fwd(q, k, v, causal=True)
    ref = fa.fa_bwd(q, k, v, out, do, lse, causal=True)
    cu = torch.tensor([0, S], dtype=torch.int32, device=cuda_device)
    got = fa.fa_varlen_bwd(q[0], k[0], v[0], out[0], do[0], lse[0].contiguous(), cu, S, causal=True)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert torch.equal(g.view(torch.int16), r[0].view(torch.int16))
