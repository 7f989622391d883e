"""GPU attention forward vs the float64 CPU oracle, element by element (needs a B200).

Small cases run the oracle over every row: they span several 128-row tiles with ragged
tails, every head dim, both dtypes, causal and not, dense and packed. The five workloads
run at full size through the same C-ABI calls the benchmark times and are checked on
sampled rows (tile edges, ends, random rows) that the oracle computes one by one.
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
import tiled_exact_attention_fwd_b200 as fa
from parity_util import assert_lse_close, assert_o_close, edge_rows

pytestmark = pytest.mark.gpu

DTYPES = [torch.float16, torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_device):
    from tiled_exact_attention_fwd_b200 import build
    build.build()
    fa.lib()
    yield
    st, where = fa.fa_device_status()
    assert st == 0, f"device status {st} at {where}"


def _run_dense(q, k, v, causal, scale=None):
    dev = torch.device("cuda:0")
    out, lse = fa.fa_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("causal", [False, True])
def test_dense_small_all_rows(D, dtype, causal):
    B, S, H = 2, 300, 3  # three query tiles, ragged tail of 44 rows
    q, k, v = fa_inputs.dense_qkv(B, S, H, D, dtype, seed=D)
    out, lse = _run_dense(q, k, v, causal)
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    assert_o_close(out, O, dtype, f"D={D} {dtype} causal={causal}")
    assert_lse_close(lse, L, f"D={D} {dtype} causal={causal}")


@pytest.mark.parametrize("S", [1, 2, 63, 127, 128, 129, 255, 257, 513])
@pytest.mark.parametrize("causal", [False, True])
def test_dense_lengths(S, causal):
    D, dtype = 128, torch.bfloat16
    q, k, v = fa_inputs.dense_qkv(1, S, 2, D, dtype, seed=S)
    out, lse = _run_dense(q, k, v, causal)
    O, L = oracle.attention_dense(q, k, v, causal=causal)
    assert_o_close(out, O, dtype, f"S={S}")
    assert_lse_close(lse, L, f"S={S}")


def test_dense_explicit_scale_and_large_scores():
    """A large scale makes the running max grow inside a row: the lazy rescale must fire."""
    D, dtype = 64, torch.float16
    q, k, v = fa_inputs.dense_qkv(1, 700, 2, D, dtype, seed=11)
    for scale in (0.02, 0.5, 1.5):
        for causal in (False, True):
            out, lse = _run_dense(q, k, v, causal, scale=scale)
            O, L = oracle.attention_dense(q, k, v, causal=causal, scale=scale)
            assert_o_close(out, O, dtype, f"scale={scale}")
            assert_lse_close(lse, L, f"scale={scale}")


def test_dense_increasing_scores_force_rescales():
    """Keys built so that each key tile raises every row's max: exercises O correction."""
    S, H, D, dtype = 640, 1, 64, torch.bfloat16
    q = torch.zeros(1, S, H, D)
    q[..., 0] = 1.0
    k = fa_inputs.normal((1, S, H, D), torch.float32, 3) * 0.1
    k[..., 0] = torch.arange(S, dtype=torch.float32)[None, :, None] * 0.125
    v = fa_inputs.normal((1, S, H, D), torch.float32, 4)
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    for causal in (False, True):
        out, lse = _run_dense(q, k, v, causal, scale=1.0)
        O, L = oracle.attention_dense(q, k, v, causal=causal, scale=1.0)
        assert_o_close(out, O, dtype, "rising")
        assert_lse_close(lse, L, "rising")


def _gold(name):
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        return json.load(f)


def _val(s):
    s = str(s)
    if s.startswith("ln("):
        return math.log(float(Fraction(s[3:-1])))
    return float(Fraction(s))


@pytest.mark.parametrize("causal", [False, True])
def test_golden_pow2_on_gpu(causal):
    """The hand-derived scale=ln2 example, head dim zero-padded to 32 (exact in bf16)."""
    g = _gold("pow2_dense.json")
    q, k, v = (torch.tensor(g[n], dtype=torch.float32) for n in ("q", "k", "v"))
    pad = lambda t: torch.nn.functional.pad(t, (0, 30)).to(torch.bfloat16).contiguous()
    out, lse = _run_dense(pad(q), pad(k), pad(v), causal, scale=math.log(2.0))
    ref = g["causal" if causal else "noncausal"]
    exp_o = np.vectorize(_val, otypes=[float])(np.array(ref["out"], dtype=object))
    exp_l = np.vectorize(_val, otypes=[float])(np.array(ref["lse"], dtype=object))
    assert_o_close(out[..., :2], exp_o, torch.bfloat16, "golden")
    assert float(out[..., 2:].abs().max()) == 0.0
    assert_lse_close(lse, exp_l, "golden")


# ----------------------------------------------------------------------------- packed
def _run_varlen(q, k, v, cu, causal, scale=None):
    dev = torch.device("cuda:0")
    lens = (cu[1:] - cu[:-1]).tolist()
    out, lse = fa.fa_varlen_fwd(q.to(dev), k.to(dev), v.to(dev), cu.to(dev), max(lens) if lens else 0,
                                causal=causal, scale=scale)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(D, causal):
    lengths = [1, 7, 128, 0, 129, 300, 64, 250, 2]
    dtype = torch.bfloat16 if D != 64 else torch.float16
    q, k, v, cu = fa_inputs.packed_qkv(lengths, 3, D, dtype, seed=D + 1)
    out, lse = _run_varlen(q, k, v, cu, causal)
    O, L = oracle.attention_varlen(q, k, v, cu, causal=causal)
    assert_o_close(out, O, dtype, f"varlen D={D}")
    assert_lse_close(lse, L, f"varlen D={D}")


def test_varlen_random_lengths_many_sequences():
    lengths = fa_inputs.random_lengths(40, 0, 400, seed=9)
    q, k, v, cu = fa_inputs.packed_qkv(lengths, 2, 128, torch.bfloat16, seed=5)
    for causal in (False, True):
        out, lse = _run_varlen(q, k, v, cu, causal)
        O, L = oracle.attention_varlen(q, k, v, cu, causal=causal)
        assert_o_close(out, O, torch.bfloat16, "varlen random")
        assert_lse_close(lse, L, "varlen random")


def test_varlen_single_sequence_matches_dense_path():
    S, H, D = 333, 2, 64
    q, k, v = fa_inputs.dense_qkv(1, S, H, D, torch.bfloat16, seed=21)
    cu = torch.tensor([0, S], dtype=torch.int32)
    for causal in (False, True):
        ov, lv = _run_varlen(q[0], k[0], v[0], cu, causal)
        od, ld = _run_dense(q, k, v, causal)
        assert torch.equal(ov.view(torch.int16), od[0].view(torch.int16))
        assert torch.equal(lv, ld[0])


@pytest.mark.parametrize("causal", [False, True])
def test_golden_pow2_varlen_on_gpu(causal):
    g = _gold("pow2_varlen.json")
    q, k, v = (torch.tensor(g[n], dtype=torch.float32) for n in ("q", "k", "v"))
    pad = lambda t: torch.nn.functional.pad(t, (0, 30)).to(torch.float16).contiguous()
    cu = torch.tensor(g["cu_seqlens"], dtype=torch.int32)
    out, lse = _run_varlen(pad(q), pad(k), pad(v), cu, causal, scale=math.log(2.0))
    ref = g["causal" if causal else "noncausal"]
    exp_o = np.vectorize(_val, otypes=[float])(np.array(ref["out"], dtype=object))
    exp_l = np.vectorize(_val, otypes=[float])(np.array(ref["lse"], dtype=object))
    assert_o_close(out[..., :2], exp_o, torch.float16, "golden varlen")
    assert_lse_close(lse, exp_l, "golden varlen")


def test_empty_varlen_is_noop():
    dev = torch.device("cuda:0")
    q = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device=dev)
    cu = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = fa.fa_varlen_fwd(q, q, q, cu, 0)
    assert out.numel() == 0


# ----------------------------------------------------------------------------- full-size workloads
def _dense_workload_sampled(name, n_random, seed=0):
    w = fa_inputs.WORKLOADS[name]
    q, k, v = fa_inputs.workload_inputs(name, seed)
    dt = fa_inputs.DTYPES[w["dtype"]]
    out, lse = _run_dense(q, k, v, w["causal"])
    B, S, H, D = q.shape
    g = fa_inputs.generator(seed + 1)
    rows = []
    for i in edge_rows(S):
        rows.append((int(torch.randint(B, (1,), generator=g)), int(torch.randint(H, (1,), generator=g)), i))
    for _ in range(n_random):
        rows.append(tuple(int(torch.randint(n, (1,), generator=g)) for n in (B, H, S)))
    rows = np.array(rows, dtype=np.int64)
    O, L = oracle.attention_dense(q, k, v, causal=w["causal"], rows=rows)
    b, h, i = rows[:, 0], rows[:, 1], rows[:, 2]
    assert_o_close(out[b, i, h], O, dt, name)
    assert_lse_close(lse[b, h, i], L, name)


def test_workload_dense_fp16_small_all_rows():
    q, k, v = fa_inputs.workload_inputs("dense_fp16_small")
    out, lse = _run_dense(q, k, v, False, scale=1.0 / math.sqrt(64))
    O, L = oracle.attention_dense(q, k, v, scale=1.0 / math.sqrt(64))
    assert_o_close(out, O, torch.float16, "dense_fp16_small")
    assert_lse_close(lse, L, "dense_fp16_small")


def test_workload_vit_bf16_sampled():
    _dense_workload_sampled("vit_bf16", 200)


def test_workload_llm_causal_bf16_sampled():
    _dense_workload_sampled("llm_causal_bf16", 200)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_workload_hdim_sweep_sampled(D):
    _dense_workload_sampled(f"hdim_sweep_fp16_d{D}", 100)


def test_workload_varlen_pipeline_all_rows():
    """unpad(q, k, v) -> packed attention -> pad, on the padded (1, 4096, 16, 128) batch."""
    case = fa_inputs.workload_inputs("varlen_bf16_32x64")
    dev = torch.device("cuda:0")
    idx = case.indices.to(dev)
    cu = case.cu_seqlens.to(dev)
    qu = fa.fa_unpad(case.q_pad.to(dev), idx)
    ku = fa.fa_unpad(case.k_pad.to(dev), idx)
    vu = fa.fa_unpad(case.v_pad.to(dev), idx)
    ou, lse = fa.fa_varlen_fwd(qu, ku, vu, cu, case.max_seqlen)
    op = fa.fa_pad(ou, idx, 1, case.total_len)
    torch.cuda.synchronize()
    # every stage against the oracle
    q_ref = oracle.unpad(case.q_pad, case.indices)
    assert torch.equal(qu.cpu().view(torch.int16), q_ref.view(torch.int16))
    O, L = oracle.attention_varlen(q_ref, oracle.unpad(case.k_pad, case.indices),
                                   oracle.unpad(case.v_pad, case.indices), case.cu_seqlens)
    assert_o_close(ou.cpu(), O, torch.bfloat16, "varlen workload")
    assert_lse_close(lse.cpu(), L, "varlen workload")
    p_ref = oracle.pad(ou.cpu(), case.indices, 1, case.total_len)
    assert torch.equal(op.cpu().view(torch.int16), p_ref.view(torch.int16))


# ----------------------------------------------------------------------------- fused packed path
def _fused_case(lengths, total_len, H, D, dtype, causal, seed, case=None):
    if case is None:
        case = fa_inputs.varlen_case(lengths, total_len, H, D, dtype, seed=seed)
    total_len = case.q_pad.shape[1]
    dev = torch.device("cuda:0")
    qp, kp, vp = case.q_pad.to(dev), case.k_pad.to(dev), case.v_pad.to(dev)
    idx, cu = case.indices.to(dev), case.cu_seqlens.to(dev)
    out = torch.full_like(qp, float("nan"))  # every element must be written
    out, lse = fa.fa_varlen_fwd_padded(qp, kp, vp, idx, cu, max(case.max_seqlen, 1), out=out, causal=causal)
    # the same path in three launches
    qu, ku, vu = fa.fa_unpad_qkv(qp, kp, vp, idx)
    ou, lu = fa.fa_varlen_fwd(qu, ku, vu, cu, max(case.max_seqlen, 1), causal=causal)
    ref_pad = fa.fa_pad(ou, idx, 1, total_len)
    torch.cuda.synchronize()
    return case, out.cpu(), lse.cpu(), ref_pad.cpu(), lu.cpu()


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (64, torch.float16), (32, torch.bfloat16),
                                     (256, torch.float16)])
@pytest.mark.parametrize("causal", [False, True])
def test_fused_padded_path(D, dtype, causal):
    lengths = [1, 70, 0, 130, 255, 64, 3]
    case, out, lse, ref_pad, ref_lse = _fused_case(lengths, 1000, 2, D, dtype, causal, seed=D)
    # identical to unpad -> varlen forward -> pad on the GPU, bit for bit
    assert torch.equal(out.view(torch.int16), ref_pad.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    # and within tolerance of the oracle; padding rows exactly zero
    O, L = oracle.attention_varlen(oracle.unpad(case.q_pad, case.indices), oracle.unpad(case.k_pad, case.indices),
                                   oracle.unpad(case.v_pad, case.indices), case.cu_seqlens, causal=causal)
    flat = out.view(-1, 2, D)
    assert_o_close(flat[case.indices], O, dtype, "fused")
    assert_lse_close(lse, L, "fused")
    mask = torch.ones(flat.shape[0], dtype=torch.bool)
    mask[case.indices] = False
    assert (flat[mask].view(torch.int16) == 0).all()


@pytest.mark.parametrize("D,dtype", [(128, torch.bfloat16), (32, torch.float16), (256, torch.bfloat16)])
@pytest.mark.parametrize("causal", [False, True])
def test_fused_right_padded(D, dtype, causal):
    """Right-padded batch: each sequence's rows form one run of consecutive padded rows, so
    32-row groups inside a run move as TMA boxes and the others as per-row copies."""
    lengths = [64, 97, 0, 32, 128, 5, 160, 33]
    case = fa_inputs.right_padded_case(lengths, 160, 2, D, dtype, seed=D + 1)
    case, out, lse, ref_pad, ref_lse = _fused_case(None, None, 2, D, dtype, causal, None, case=case)
    assert torch.equal(out.view(torch.int16), ref_pad.view(torch.int16))
    assert torch.equal(lse, ref_lse)
    O, L = oracle.attention_varlen(oracle.unpad(case.q_pad, case.indices), oracle.unpad(case.k_pad, case.indices),
                                   oracle.unpad(case.v_pad, case.indices), case.cu_seqlens, causal=causal)
    flat = out.view(-1, 2, D)
    assert_o_close(flat[case.indices], O, dtype, "fused right-padded")
    assert_lse_close(lse, L, "fused right-padded")
    mask = torch.ones(flat.shape[0], dtype=torch.bool)
    mask[case.indices] = False
    assert (flat[mask].view(torch.int16) == 0).all()


def test_fused_workload_32x64():
    w = fa_inputs.WORKLOADS["varlen_bf16_32x64"]
    case, out, lse, ref_pad, ref_lse = _fused_case(w["lengths"], w["total_len"], w["H"], w["D"], torch.bfloat16,
                                                   False, seed=0)
    assert torch.equal(out.view(torch.int16), ref_pad.view(torch.int16))
    assert torch.equal(lse, ref_lse)


def test_fused_edge_cases():
    dev = torch.device("cuda:0")
    # no valid token: all zeros
    x = fa_inputs.normal((1, 300, 2, 64), torch.bfloat16, 1).to(dev)
    idx = torch.zeros(0, dtype=torch.int64, device=dev)
    cu = torch.zeros(1, dtype=torch.int32, device=dev)
    out, _ = fa.fa_varlen_fwd_padded(x, x, x, idx, cu, 0, out=torch.full_like(x, 7.0))
    assert float(out.abs().max()) == 0.0
    # no padding at all: equals the plain packed call
    case, out, lse, ref_pad, ref_lse = _fused_case([100, 156], 256, 2, 64, torch.bfloat16, True, seed=3)
    assert torch.equal(out.view(torch.int16), ref_pad.view(torch.int16))
