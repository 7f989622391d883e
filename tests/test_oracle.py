"""Pins of the float64 CPU oracle to facts the pages and the mathematics fix (CPU only).

Every check here compares the oracle with something other than itself: hand-derived
worked examples (tests/golden), closed forms, invariants of softmax attention, a library
routine that computes the same thing (torch's fp64 scaled_dot_product_attention on the
CPU), and the pages' blockwise online-softmax merge.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import fa_inputs
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _val(s):
    s = str(s)
    if s.startswith("ln(") and s.endswith(")"):
        return math.log(float(Fraction(s[3:-1])))
    return float(Fraction(s))


def _arr(nested):
    return np.vectorize(_val, otypes=[float])(np.array(nested, dtype=object))


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed):
    return fa_inputs.normal(shape, torch.float32, seed).double()


# ----------------------------------------------------------------------------- golden cases
@pytest.mark.parametrize("causal", [False, True])
def test_golden_pow2_dense(causal):
    g = _load("pow2_dense.json")
    q, k, v = (torch.tensor(g[n], dtype=torch.float64) for n in ("q", "k", "v"))
    O, L = oracle.attention_dense(q, k, v, scale=_val(g["scale"]), causal=causal)
    ref = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(O, _arr(ref["out"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, _arr(ref["lse"]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_golden_pow2_varlen(causal):
    g = _load("pow2_varlen.json")
    q, k, v = (torch.tensor(g[n], dtype=torch.float64) for n in ("q", "k", "v"))
    O, L = oracle.attention_varlen(q, k, v, g["cu_seqlens"], scale=_val(g["scale"]), causal=causal)
    ref = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(O, _arr(ref["out"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, _arr(ref["lse"]), rtol=0, atol=1e-13)


def test_golden_pad_unpad_bytes():
    g = _load("pad_unpad_bytes.json")
    x = torch.tensor(g["rows"], dtype=torch.uint8).reshape(1, 6, 1, 4)
    idx = torch.tensor(g["indices"], dtype=torch.int64)
    u = oracle.unpad(x, idx)
    assert u.reshape(3, 4).tolist() == g["unpad"]
    p = oracle.pad(u, idx, 1, 6)
    assert p.reshape(6, 4).tolist() == g["pad_of_unpad"]


# ----------------------------------------------------------------------------- softmax facts
@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    S, H, D = 37, 2, 16
    q, k, v = (_rand((S, H, D), s) * 3 for s in (1, 2, 3))
    tok, head, lo, hi = oracle.dense_row_spec(1, S, H, None, causal)
    _, _, P = oracle.attention_rows(q, k, v, tok, head, lo, hi, causal=causal, want_probs=True)
    sums = P.sum(axis=1)
    assert np.max(np.abs(sums - 1.0)) < 1e-12
    assert (P >= 0).all()
    if causal:  # keys after the query carry exactly zero weight
        pos = tok - lo
        for r in range(P.shape[0]):
            assert (P[r, pos[r] + 1:] == 0).all()


@pytest.mark.parametrize("block", [1, 3, 7, 16, 64, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_merge_equals_full_softmax(block, causal):
    """The pages' blockwise merge (running max m and sum d) reproduces the full softmax."""
    S, D = 53, 24
    q, k, v = (_rand((S, 1, D), s) * 2 for s in (4, 5, 6))
    O, L = oracle.attention_dense(q[None], k[None], v[None], causal=causal)
    Ob, Lb = oracle.online_softmax_attention(q[:, 0].numpy(), k[:, 0].numpy(), v[:, 0].numpy(),
                                             block, causal=causal)
    np.testing.assert_allclose(Ob, O[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lb, L[0, 0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("zero", ["q", "k"])
def test_uniform_scores_give_mean_of_v(causal, zero):
    B, S, H, D = 2, 19, 3, 8
    q, k, v = (_rand((B, S, H, D), s) for s in (7, 8, 9))
    if zero == "q":
        q = torch.zeros_like(q)
    else:
        k = torch.zeros_like(k)
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    if causal:
        counts = torch.arange(1, S + 1, dtype=torch.float64)
        mean = v.cumsum(dim=1) / counts[None, :, None, None]
        lse = np.log(counts.numpy())[None, None, :].repeat(B, 0).repeat(H, 1)
    else:
        mean = v.mean(dim=1, keepdim=True).expand(B, S, H, D)
        lse = np.full((B, H, S), math.log(S))
    np.testing.assert_allclose(O, mean.numpy(), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, lse, rtol=0, atol=1e-13)


def test_causal_row_zero_is_v0():
    B, S, H, D = 2, 11, 2, 16
    q, k, v = (_rand((B, S, H, D), s) for s in (10, 11, 12))
    O, L = oracle.attention_dense(q, k, v, causal=True, scale=0.3)
    assert np.array_equal(O[:, 0], v[:, 0].numpy())  # weight exactly 1
    for b in range(B):
        for h in range(H):
            s0 = 0.3 * math.fsum((q[b, 0, h] * k[b, 0, h]).tolist())
            assert abs(L[b, h, 0] - s0) < 1e-13


def test_single_key_gives_v_and_score():
    H, D = 3, 8
    q, k, v = (_rand((1, 1, H, D), s) for s in (13, 14, 15))
    O, L = oracle.attention_dense(q, k, v, scale=0.5)
    assert np.array_equal(O[0, 0], v[0, 0].numpy())
    for h in range(H):
        assert abs(L[0, h, 0] - 0.5 * math.fsum((q[0, 0, h] * k[0, 0, h]).tolist())) < 1e-13


def test_two_keys_logistic_closed_form():
    """With two keys the weights are the logistic function of the score difference."""
    H, D = 2, 8
    q, k, v = (_rand((1, 2, H, D), s) * 2 for s in (16, 17, 18))
    sc = 0.7
    O, L = oracle.attention_dense(q, k, v, scale=sc)
    for i in range(2):
        for h in range(H):
            s0 = sc * math.fsum((q[0, i, h] * k[0, 0, h]).tolist())
            s1 = sc * math.fsum((q[0, i, h] * k[0, 1, h]).tolist())
            w0 = 1.0 / (1.0 + math.exp(s1 - s0))
            w1 = 1.0 / (1.0 + math.exp(s0 - s1))
            exp_o = w0 * v[0, 0, h].numpy() + w1 * v[0, 1, h].numpy()
            np.testing.assert_allclose(O[0, i, h], exp_o, rtol=0, atol=1e-13)
            assert abs(L[0, h, i] - np.logaddexp(s0, s1)) < 1e-13


def test_identical_keys_give_mean_of_v():
    S, H, D = 23, 2, 8
    q, v = _rand((1, S, H, D), 19), _rand((1, S, H, D), 20)
    k = _rand((1, 1, H, D), 21).expand(1, S, H, D).contiguous()
    O, _ = oracle.attention_dense(q, k, v)
    np.testing.assert_allclose(O, v.mean(dim=1, keepdim=True).expand_as(v).numpy(), atol=1e-13)


def test_kv_permutation_invariance_noncausal():
    S, H, D = 29, 2, 16
    q, k, v = (_rand((1, S, H, D), s) for s in (22, 23, 24))
    perm = torch.randperm(S, generator=fa_inputs.generator(5))
    O1, L1 = oracle.attention_dense(q, k, v)
    O2, L2 = oracle.attention_dense(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)


def test_affine_in_v():
    S, H, D = 17, 2, 8
    q, k, v = (_rand((1, S, H, D), s) for s in (25, 26, 27))
    a, b = 2.5, -1.25
    for causal in (False, True):
        O1, _ = oracle.attention_dense(q, k, v, causal=causal)
        O2, _ = oracle.attention_dense(q, k, a * v + b, causal=causal)
        np.testing.assert_allclose(O2, a * O1 + b, atol=1e-12)


def test_lse_shift_by_constant_score():
    """Adding c*q to every key shifts each score by c|q|^2*scale: LSE shifts, O does not."""
    S, H, D = 13, 1, 8
    q = _rand((1, 1, H, D), 28).expand(1, S, H, D).contiguous()
    k, v = _rand((1, S, H, D), 29), _rand((1, S, H, D), 30)
    c, sc = 0.75, 0.4
    O1, L1 = oracle.attention_dense(q, k, v, scale=sc)
    O2, L2 = oracle.attention_dense(q, k + c * q, v, scale=sc)
    shift = sc * c * float((q[0, 0, 0] ** 2).sum())
    np.testing.assert_allclose(O1, O2, atol=1e-12)
    np.testing.assert_allclose(L2 - L1, shift, atol=1e-12)


# ----------------------------------------------------------------------------- library routine
@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_fp64(causal):
    B, S, H, D = 2, 45, 3, 32
    q, k, v = (_rand((B, S, H, D), s) for s in (31, 32, 33))
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2), is_causal=causal).transpose(1, 2)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(D)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_row_sample_matches_full():
    B, S, H, D = 2, 40, 3, 16
    q, k, v = (_rand((B, S, H, D), s) for s in (34, 35, 36))
    for causal in (False, True):
        O, L = oracle.attention_dense(q, k, v, causal=causal)
        rows = np.array([[0, 0, 0], [1, 2, 39], [0, 1, 17], [1, 0, 5]])
        Or, Lr = oracle.attention_dense(q, k, v, causal=causal, rows=rows)
        for r, (b, h, i) in enumerate(rows):
            assert np.array_equal(Or[r], O[b, i, h])
            assert Lr[r] == L[b, h, i]


# ----------------------------------------------------------------------------- varlen
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_per_sequence_dense(causal):
    lengths = [5, 1, 17, 9, 0, 30]
    H, D = 2, 16
    q, k, v, cu = fa_inputs.packed_qkv(lengths, H, D, torch.float32, seed=3)
    q, k, v = q.double(), k.double(), v.double()
    O, L = oracle.attention_varlen(q, k, v, cu, causal=causal)
    for s, n in enumerate(lengths):
        a, b = int(cu[s]), int(cu[s + 1])
        if n == 0:
            continue
        Od, Ld = oracle.attention_dense(q[None, a:b], k[None, a:b], v[None, a:b], causal=causal)
        np.testing.assert_allclose(O[a:b], Od[0], atol=1e-13)
        np.testing.assert_allclose(L[:, a:b], Ld[0], atol=1e-13)


def test_varlen_single_sequence_equals_dense():
    S, H, D = 33, 2, 8
    q, k, v = (_rand((1, S, H, D), s) for s in (37, 38, 39))
    for causal in (False, True):
        O, L = oracle.attention_dense(q, k, v, causal=causal)
        Ov, Lv = oracle.attention_varlen(q[0], k[0], v[0], [0, S], causal=causal)
        np.testing.assert_allclose(Ov, O[0], atol=1e-13)
        np.testing.assert_allclose(Lv, L[0], atol=1e-13)


# ----------------------------------------------------------------------------- unpad / pad
def test_unpad_pad_round_trip():
    case = fa_inputs.varlen_case([7, 3, 12], 40, 3, 8, torch.bfloat16, seed=2)
    u = oracle.unpad(case.q_pad, case.indices)
    assert u.shape == (22, 3, 8)
    flat = case.q_pad.view(-1, 3, 8)
    assert torch.equal(u.view(torch.int16), flat[case.indices].view(torch.int16))
    p = oracle.pad(u, case.indices, 1, 40)
    mask = torch.zeros(40, dtype=torch.bool)
    mask[case.indices] = True
    assert torch.equal(p[0][mask].view(torch.int16), flat[mask].view(torch.int16))
    assert (p[0][~mask].view(torch.int16) == 0).all()


def test_unpad_pad_reject_out_of_range():
    x = torch.zeros(1, 4, 1, 8, dtype=torch.float16)
    with pytest.raises(ValueError):
        oracle.unpad(x, torch.tensor([0, 4]))
    with pytest.raises(ValueError):
        oracle.pad(torch.zeros(2, 1, 8, dtype=torch.float16), torch.tensor([-1, 2]), 1, 4)


def test_empty_inputs():
    x = torch.zeros(1, 4, 2, 8, dtype=torch.bfloat16)
    assert oracle.unpad(x, torch.zeros(0, dtype=torch.int64)).shape == (0, 2, 8)
    p = oracle.pad(torch.zeros(0, 2, 8, dtype=torch.bfloat16), torch.zeros(0, dtype=torch.int64), 1, 4)
    assert (p.view(torch.int16) == 0).all()


def test_inputs_are_deterministic():
    a = fa_inputs.dense_qkv(1, 8, 2, 16, torch.bfloat16, seed=4)
    b = fa_inputs.dense_qkv(1, 8, 2, 16, torch.bfloat16, seed=4)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    c = fa_inputs.varlen_case([64] * 32, 4096, 16, 128, torch.bfloat16)
    assert c.nnz == 2048 and int(c.cu_seqlens[-1]) == 2048
    assert torch.all(c.indices[1:] > c.indices[:-1])
