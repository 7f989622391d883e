"""Pins of the float64 backward oracle (CPU): finite differences of the forward oracle,
torch float64 autograd, and closed forms / invariants of the softmax derivative."""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_finite_differences_of_the_forward_oracle(causal):
    """d(sum(O * G))/dx by central differences of the (C, float64) forward oracle."""
    B, S, H, D = 1, 9, 2, 4
    q, k, v, g = (_rand((B, S, H, D), s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle.attention_backward(q, k, v, g, causal=causal)
    eps = 1e-5
    rng = np.random.default_rng(5)

    def loss(qq, kk, vv):
        O, _ = oracle.attention_dense(qq, kk, vv, causal=causal)
        return float((O * g.numpy()).sum())

    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in (B, S, H, D))
            args = {"q": q.clone(), "k": k.clone(), "v": v.clone()}
            args[name][idx] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * eps
            down = loss(args["q"], args["k"], args["v"])
            fd = (up - down) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_fp64(causal):
    B, S, H, D = 2, 13, 2, 8
    q, k, v, g = (_rand((B, S, H, D), s) for s in (11, 12, 13, 14))
    qt, kt, vt = (t.clone().transpose(1, 2).requires_grad_() for t in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)
    out.backward(g.transpose(1, 2))
    dq, dk, dv = oracle.attention_backward(q, k, v, g, causal=causal)
    for ours, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        np.testing.assert_allclose(ours, ref.transpose(1, 2).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_gradients_sum_to_zero(causal):
    """Each row of dZ sums to zero (softmax is shift invariant), so sum_j dK_j = 0."""
    q, k, v, g = (_rand((1, 20, 1, 6), s) for s in (21, 22, 23, 24))
    _, dk, _ = oracle.attention_backward(q, k, v, g, causal=causal)
    assert np.abs(dk.sum(axis=1)).max() < 1e-12


def test_single_key_closed_form():
    """One key: the softmax weight is 1 whatever the score, so dV = dO and dQ = dK = 0."""
    q, k, v, g = (_rand((1, 1, 1, 5), s) for s in (31, 32, 33, 34))
    dq, dk, dv = oracle.attention_backward(q, k, v, g)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    np.testing.assert_array_equal(dv, g.numpy())


def test_causal_row_zero_has_no_query_gradient():
    q, k, v, g = (_rand((1, 7, 1, 4), s) for s in (41, 42, 43, 44))
    dq, _, _ = oracle.attention_backward(q, k, v, g, causal=True)
    assert np.abs(dq[0, 0]).max() == 0


def test_uniform_scores_closed_form():
    """Q = 0 (non-causal): every weight is 1/S, so dV_j = mean_i dO_i and dK = 0."""
    S = 10
    q = torch.zeros((1, S, 1, 4), dtype=torch.float64)
    k, v, g = (_rand((1, S, 1, 4), s) for s in (51, 52, 53))
    dq, dk, dv = oracle.attention_backward(q, k, v, g)
    np.testing.assert_allclose(dv[0, :, 0], np.tile(g.numpy()[0, :, 0].mean(axis=0), (S, 1)), atol=1e-14)
    assert np.abs(dk).max() < 1e-15


def test_head_subset_matches_full():
    q, k, v, g = (_rand((2, 6, 3, 4), s) for s in (61, 62, 63, 64))
    full = oracle.attention_backward(q, k, v, g, causal=True)
    part = oracle.attention_backward(q, k, v, g, causal=True, heads=[(1, 2), (0, 1)])
    for (b, h), grads in part.items():
        for a, f in zip(grads, full):
            np.testing.assert_array_equal(a, f[b, :, h])


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_backward_equals_per_sequence_dense(causal):
    """The packed gradients are those of each sequence alone (zero-length sequences allowed)."""
    lengths = [5, 0, 17, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    total, H, D = int(cu[-1]), 2, 8
    q, k, v, g = (_rand((total, H, D), s) for s in (71, 72, 73, 74))
    dq, dk, dv = oracle.attention_varlen_backward(q, k, v, g, cu, causal=causal)
    for s0, s1 in zip(cu[:-1], cu[1:]):
        if s1 == s0:
            continue
        ref = oracle.attention_backward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], g[None, s0:s1], causal=causal)
        for a, r in zip((dq, dk, dv), ref):
            np.testing.assert_array_equal(a[s0:s1], r[0])
