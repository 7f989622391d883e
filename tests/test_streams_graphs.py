"""Launch properties of the C ABI on the GPU: results are deterministic, calls on side streams
and concurrent streams give the same bits, and every entry point can be captured into a CUDA
graph (no allocation or synchronisation inside a call) and replayed."""
import pytest
import torch

import fa_inputs

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.dtype in (torch.bfloat16, torch.float16) else t.view(torch.int32)


def _dense(dev, seed=0, B=2, S=300, H=4, D=128, dtype=torch.bfloat16):
    return [t.to(dev) for t in fa_inputs.dense_qkv(B, S, H, D, dtype, seed=seed)]


def test_forward_and_backward_are_deterministic(cuda_device):
    import tiled_exact_attention_fwd_b200 as fa
    q, k, v = _dense(cuda_device)
    do = fa_inputs.normal(tuple(q.shape), q.dtype, seed=9).to(cuda_device)
    o1, l1 = fa.fa_fwd(q, k, v, causal=True)
    o2, l2 = fa.fa_fwd(q, k, v, causal=True)
    g1 = fa.fa_bwd(q, k, v, o1, do, l1, causal=True)
    g2 = fa.fa_bwd(q, k, v, o1, do, l1, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(_bits(o1), _bits(o2)) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(_bits(a), _bits(b))


def test_side_streams_run_concurrently_and_agree(cuda_device):
    import tiled_exact_attention_fwd_b200 as fa
    inputs = [_dense(cuda_device, seed=s) for s in range(3)]
    ref = [fa.fa_fwd(*x, causal=bool(i % 2))[0] for i, x in enumerate(inputs)]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(device=cuda_device) for _ in inputs]
    outs = []
    for i, (x, st) in enumerate(zip(inputs, streams)):
        st.wait_stream(torch.cuda.current_stream(cuda_device))
        with torch.cuda.stream(st):
            out = torch.empty_like(x[0])
            fa.fa_fwd(*x, out=out, causal=bool(i % 2), return_lse=False, stream=st)
            outs.append(out)
    torch.cuda.synchronize()
    for a, b in zip(outs, ref):
        assert torch.equal(_bits(a), _bits(b))
    assert fa.fa_device_status()[0] == 0


def test_cuda_graph_capture_and_replay(cuda_device):
    import tiled_exact_attention_fwd_b200 as fa
    dev = cuda_device
    q, k, v = _dense(dev, seed=4)
    do = fa_inputs.normal(tuple(q.shape), q.dtype, seed=5).to(dev)
    case = fa_inputs.varlen_case([5, 130, 64, 1], 256, 2, 64, torch.float16, seed=6)
    qp, kp, vp = case.q_pad.to(dev), case.k_pad.to(dev), case.v_pad.to(dev)
    idx, cu = case.indices.to(dev), case.cu_seqlens.to(dev)
    kc_h, vc_h, table_h = fa_inputs.paged_kv(k.cpu(), v.cpu(), 32, seed=7)
    kc, vc, table = kc_h.to(dev), vc_h.to(dev), table_h.to(dev)

    out = torch.empty_like(q)
    lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    delta = torch.empty_like(lse)
    outp = torch.empty_like(qp)
    lsep = torch.empty((2, case.nnz), device=dev, dtype=torch.float32)
    outg = torch.empty_like(q)

    def body():
        fa.fa_fwd(q, k, v, out=out, lse=lse, causal=True)
        fa.fa_bwd(q, k, v, out, do, lse, dq=dq, dk=dk, dv=dv, delta=delta, causal=True)
        fa.fa_varlen_fwd_padded(qp, kp, vp, idx, cu, 130, out=outp, lse=lsep)
        fa.fa_fwd_paged(q, kc, vc, table, out=outg, causal=True, return_lse=False)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        body()  # warm-up: per-device function attributes are set outside the capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (out, lse, dq, dk, dv, outp, lsep, outg)]
    for t in (out, dq, dk, dv, outp, outg):
        t.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        got = (out, lse, dq, dk, dv, outp, lsep, outg)
        for a, b in zip(got, ref):
            assert torch.equal(_bits(a), _bits(b))
    assert fa.fa_device_status()[0] == 0
