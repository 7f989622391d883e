"""Benchmark of the attention forward path on B200 (one JSON line on rank 0).

Workload timed as `value`: causal bf16 attention forward, B=1 H=32 S=8192 D=128
(the sequence-length-8192 causal case, scale 1/sqrt(128)), inputs N(0,1) from a seed,
resident in HBM. q, k, v, out total 256 MiB, larger than the 126 MB L2, so no flush is
needed between steps. One step = one fa_fwd launch.

Also reported on the same line:
  e2e          the same TFLOPS through the C ABI with pinned HOST buffers: each step copies
               q, k, v to the device, runs fa_fwd, and copies out + lse back.
  varlen       the packed path at 32 sequences x 64 tokens, H=16, D=128, bf16, padded batch
               (1, 4096, 16, 128): unpad(q), unpad(k), unpad(v), varlen forward, pad(out),
               in microseconds per call (and per component).
  roofline     tensor-bound: achieved TFLOPS of the attention kernel vs the measured bf16 peak.
  cpu_baseline the float64 CPU oracle on a bounded sample of the same workload.

  configs      every workload of the pages (small dense, packed 32x64, ViT, the causal 8192
               case, the head-dim sweep at 4096): time per call or TFLOPS, and each one's
               roofline: tensor-bound (FLOPs / measured bf16 peak) or exp-bound (one exp2 per
               visible score / MUFU rate of 16 per clock per SM at the sampled SM clock).

Launch: `python bench.py [--gpus N --steps K --warmup W]`. With N > 1 and no torchrun
environment, bench.py starts itself under torch.distributed.run with N local ranks; every
rank runs the same per-GPU workload (replicas: weak scaling, no collective on the data path)
and the time is the max over ranks.
`--impl reference` times the float64 CPU oracle (the only reference this path has).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import fa_inputs  # noqa: E402

METRIC = "attention fwd TFLOPS and % of B200 tensor-core peak; varlen µs/call"
WORKLOAD = "llm_causal_bf16"
KERNEL_SOURCES = ["tiled_exact_attention_fwd_b200/csrc/fa_fwd_kernel.cuh", "tiled_exact_attention_fwd_b200/csrc/fa_ptx.cuh",
                  "tiled_exact_attention_fwd_b200/csrc/fa_sync.cuh", "tiled_exact_attention_fwd_b200/csrc/fa_seq.cuh"]


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    """(bf16 burst TF/s, HBM GB/s, kind, bf16 sustained TF/s) from MEASURED_PEAKS.json, else fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured",
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])))
    return 1590.0, 6650.0, "fallback", 1400.0


# A timed region longer than this runs into the 1 kW power cap on B200 (measured: the
# causal forward loses ~8% between 100- and 200-launch windows), so it is compared with
# the sustained GEMM figure rather than the burst one.
BURST_WINDOW_MS = 50.0


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every ~2 ms while running."""

    REASONS = {
        0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
        0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        bins = {}
        for mhz in self.samples:
            bins[str(int(mhz) // 15 * 15)] = bins.get(str(int(mhz) // 15 * 15), 0) + 1
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "mhz_bins_15": bins}


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int, device):
    torch.cuda.synchronize(device)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
    torch.cuda.synchronize(device)


# ----------------------------------------------------------------------------- CPU oracle sample
def oracle_sample(budget_s: float = 12.0, threads: int = 0, max_heads: int = 0):
    """Times the float64 oracle on whole heads of the causal workload (every query row).

    Heads are added until about `budget_s` of CPU time is spent (all 32 heads = the whole
    workload). Returns (tflops, seconds, heads, flops, threads_used). Query row i (causal)
    costs 4*D*(i+1) flops: 2*D per visible key for q.k and 2*D for p*v, which sums to the
    4*B*H*S*S*D/2 convention of the GPU figure up to the diagonal term.
    """
    import numpy as np

    import oracle
    w = fa_inputs.WORKLOADS[WORKLOAD]
    B, S, H, D = w["B"], w["S"], w["H"], w["D"]
    nth = threads if threads > 0 else oracle.max_threads()
    H_max = max_heads if max_heads > 0 else H
    q, k, v = (fa_inputs.normal((B, S, H_max, D), torch.bfloat16, 100 + s) for s in range(3))
    row_flops = float(sum(4 * D * (i + 1) for i in range(S)))

    def run(h0, nh):
        rows = np.stack([np.zeros(nh * S, np.int64), np.repeat(np.arange(h0, h0 + nh), S),
                         np.tile(np.arange(S), nh)], axis=1)
        t0 = time.perf_counter()
        oracle.attention_dense(q, k, v, causal=w["causal"], rows=rows, nthreads=nth)
        return time.perf_counter() - t0

    dt = run(0, 1)
    heads = 1
    if dt < budget_s and H_max > 1:
        more = int(min(H_max - 1, max(0, (budget_s - dt) / dt)))
        if more > 0:
            dt += run(1, more)
            heads += more
    flops = row_flops * heads
    return flops / dt / 1e12, dt, heads, flops, nth


# ----------------------------------------------------------------------------- our arm
def run_ours(args):
    ws, rank, local = dist_info()
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import tiled_exact_attention_fwd_b200 as fa
    fa.lib()  # raises if the CUDA library is missing: there is no fallback

    w = fa_inputs.WORKLOADS[WORKLOAD]
    B, S, H, D, causal = w["B"], w["S"], w["H"], w["D"], w["causal"]
    dt = fa_inputs.DTYPES[w["dtype"]]
    q_h, k_h, v_h = fa_inputs.dense_qkv(B, S, H, D, dt, seed=rank)
    q, k, v = q_h.to(device), k_h.to(device), v_h.to(device)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), device=device, dtype=torch.float32)
    flops = fa.attention_flops(B, H, S, S, D, causal)
    stream = torch.cuda.current_stream(device)

    def step():
        fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)

    for _ in range(args.warmup):
        step()
    barrier(ws, device)
    sampler = ClockSampler(device.index)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize(device)
    barrier(ws, device)
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, ws, device)
    st, where = fa.fa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where}")
    value = flops * ws / (ms * 1e-3) / 1e12
    kernel_tflops = flops / (ms_local * 1e-3) / 1e12
    # The timed region is short (K steps of ~0.5 ms): NVML gets only a sample or two in it. The
    # same step repeated for ~150 ms right after it, under its own sampler, shows where the
    # clocks sit while this kernel runs (informational; the timed value is the K-step region's).
    repeat_clocks = None
    if not args.only_main:
        reps = max(1, int(150.0 / max(ms_local, 1e-3)))
        rs = ClockSampler(device.index)
        with rs:
            for _ in range(reps):
                step()
            torch.cuda.synchronize(device)
        repeat_clocks = rs.summary()
        repeat_clocks["steps"] = reps
    if args.only_main:  # short run of the main kernel alone (profiling)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": round(value, 2), "unit": "TFLOPS",
                              "ms_per_step": round(ms, 4), "steps": args.steps, "only_main": True}), flush=True)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    # ---- end to end through the C ABI with pinned host buffers. Every step copies its
    # q, k, v in from pinned host memory, runs fa_fwd and copies out and lse back. Steps are
    # pipelined over two device buffer sets and three streams (copy in, compute, copy out),
    # so step i+1's inputs cross PCIe while step i computes and step i-1's outputs return.
    qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
    sets = [(q, k, v, out, lse)] + [tuple(torch.empty_like(t) for t in (q, k, v, out, lse))]
    hosts = [(torch.empty(q_h.shape, dtype=dt).pin_memory(), torch.empty((B, H, S), dtype=torch.float32).pin_memory())
             for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("in", "comp", "out")}

    def e2e_steps_run(n, start_ev, end_ev):
        start_ev.record(s_in)
        for i in range(n):
            b = i % 2
            dq_, dk_, dv_, do_, dl_ = sets[b]
            ho, hl = hosts[b]
            if i >= 2:
                s_in.wait_event(ev["comp"][b])   # step i-2 no longer reads these inputs
            with torch.cuda.stream(s_in):
                dq_.copy_(qp, non_blocking=True)
                dk_.copy_(kp, non_blocking=True)
                dv_.copy_(vp, non_blocking=True)
            ev["in"][b].record(s_in)
            stream.wait_event(ev["in"][b])
            if i >= 2:
                stream.wait_event(ev["out"][b])  # step i-2's outputs have left these buffers
            fa.fa_fwd(dq_, dk_, dv_, out=do_, lse=dl_, causal=causal, stream=stream)
            ev["comp"][b].record(stream)
            s_out.wait_event(ev["comp"][b])
            with torch.cuda.stream(s_out):
                ho.copy_(do_, non_blocking=True)
                hl.copy_(dl_, non_blocking=True)
            ev["out"][b].record(s_out)
        s_in.wait_stream(s_out)
        s_in.wait_stream(stream)
        end_ev.record(s_in)

    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize(device)
    e2e_steps_run(2, torch.cuda.Event(), torch.cuda.Event())  # warm-up
    torch.cuda.synchronize(device)
    barrier(ws, device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps_run(e2e_steps, t0, t1)
    torch.cuda.synchronize(device)
    barrier(ws, device)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1) / e2e_steps, ws, device)
    h2d = 3 * q_h.numel() * q_h.element_size()
    d2h = hosts[0][0].numel() * hosts[0][0].element_size() + hosts[0][1].numel() * 4
    del sets[1:]

    # the other legs run under a second clock sampler (their timings use its median clock)
    legs_sampler = ClockSampler(device.index)
    legs_sampler.__enter__()

    # ---- the backward pass of the same problem (recomputation from the saved LSE)
    backward = run_backward_leg(fa, device, stream, q, k, v, out, lse, causal, args.warmup, rank)

    # ---- the same problem with K/V in page pools (block table), per page size
    paged = run_paged_leg(fa, device, stream, q, k_h, v_h, causal, flops, args.warmup, rank)

    # ---- packed path (unpad x3, varlen forward, pad), microseconds per call
    varlen = run_varlen_leg(fa, device, stream, max(args.steps, 20), args.warmup, ws)
    padding = run_padding_hbm_leg(fa, device, stream, 20)
    del qp, kp, vp, hosts

    # ---- every workload of the pages, each against its own roofline
    main_clocks = sampler.summary()
    mhz = main_clocks.get("sm_mhz") or main_clocks.get("sm_max_mhz") or 1965.0
    configs = run_configs_leg(fa, device, stream, args.warmup, float(mhz), ms_local, varlen)
    legs_sampler.__exit__()

    peak_burst, peak_bw, peak_kind, peak_sust = load_peaks()
    clocks = main_clocks
    clocks["main_step_repeated"] = repeat_clocks
    clocks["other_legs"] = legs_sampler.summary()
    timed_ms = ms_local * args.steps
    long_region = timed_ms > BURST_WINDOW_MS or "sw_power_cap" in clocks.get("reasons", [])
    peak_tf = peak_sust if long_region else peak_burst
    peak_label = (f"{peak_kind} bf16 dense, {'sustained' if long_region else 'burst'} "
                  f"(timed region {timed_ms:.0f} ms{', sw_power_cap seen' if 'sw_power_cap' in clocks.get('reasons', []) else ''})")
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1))",
        "config": {"workload": "causal attention fwd, B=1 H=32 S=8192 D=128 bf16, scale 1/sqrt(128)",
                   "B": B, "H": H, "S": S, "D": D, "causal": causal,
                   "flops_per_step": flops, "l2": "inputs larger than L2 (q,k,v,out = 256 MiB); no flush",
                   "parallelism": f"replicas x{ws} (independent per-GPU problems)"},
        "gpu_launches": args.steps,
        "e2e": {"value": round(flops * ws / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipeline": "copy-in / fa_fwd / copy-out on three streams, two buffer sets"},
        "roofline": {"bound": "tensor", "achieved": round(kernel_tflops, 2), "peak": peak_tf,
                     "unit": "TFLOP/s", "frac": round(kernel_tflops / peak_tf, 4),
                     "peak_kind": peak_label, "frac_vs_burst": round(kernel_tflops / peak_burst, 4),
                     "frac_vs_sustained": round(kernel_tflops / peak_sust, 4),
                     "kernel": "fa_fwd_kernel<128,bf16,causal>",
                     "traffic": recorded_traffic("fa_fwd_kernel_d128_bf16_causal")},
        "configs": configs,
        "varlen": varlen,
        "paged": paged,
        "backward": backward,
        "unpad_pad_hbm": padding,
        "clocks": clocks,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tf, secs, nheads, fl, nth = oracle_sample()
        result["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOPS", "cores": nth, "kind": "oracle",
                                  "sample": f"all 8192 query rows of {nheads} of the 32 heads (causal, S=8192, "
                                            f"D=128), {fl:.3g} flops in {secs:.1f} s, float64 OpenMP"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_backward_leg(fa, device, stream, q, k, v, out, lse, causal, warmup, rank, iters=10):
    """fa_bwd on the main workload: TFLOPS by the usual 2.5x-forward convention."""
    B, S, H, D = q.shape
    do = fa_inputs.normal(tuple(q.shape), q.dtype, seed=rank + 100).to(device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    delta = torch.empty((B, H, S), device=device, dtype=torch.float32)
    fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)

    ms = _time_bwd(fa, device, stream, q, k, v, out, do, lse, dq, dk, dv, delta, causal, warmup, iters)
    flops = fa.attention_bwd_flops(B, H, S, D, causal)
    peak_burst, _, _, _ = load_peaks()
    tf = flops / (ms * 1e-3) / 1e12
    res = {"what": "fa_bwd (delta, dK/dV and dQ kernels) on the main workload; FLOPs = 2.5x the forward's "
                   "(five S x S x D products; the dQ kernel recomputes two of them, not counted)",
           "ms": round(ms, 4), "tflops": round(tf, 1), "frac_vs_burst": round(tf / peak_burst, 4),
           "launches": 3 * iters}
    # the largest head dim of the head-dim sweep (page "FlashAttention性能调优：block_size和head_dim怎么选？",
    # head_dim measurements at seq_len 4096)
    B2, S2, H2, D2 = 1, 4096, 16, 256
    q2, k2, v2 = (t.to(device) for t in fa_inputs.dense_qkv(B2, S2, H2, D2, torch.float16, seed=rank + 200))
    do2 = fa_inputs.normal((B2, S2, H2, D2), torch.float16, seed=rank + 300).to(device)
    out2, lse2 = fa.fa_fwd(q2, k2, v2, causal=True, stream=stream)
    g2 = [torch.empty_like(q2) for _ in range(3)]
    delta2 = torch.empty((B2, H2, S2), device=device, dtype=torch.float32)
    ms2 = _time_bwd(fa, device, stream, q2, k2, v2, out2, do2, lse2, *g2, delta2, True, warmup, iters)
    tf2 = fa.attention_bwd_flops(B2, H2, S2, D2, True) / (ms2 * 1e-3) / 1e12
    res["hdim256"] = {"what": "fa_bwd at B1 H16 S4096 D256 causal fp16 (delta, dV, dK and dQ kernels: one "
                              "accumulator per kernel at D = 256); FLOPs = 2.5x the forward's (the kernels "
                              "compute eight S x S x D products, three recomputed and not counted)",
                      "ms": round(ms2, 4), "tflops": round(tf2, 1), "frac_vs_burst": round(tf2 / peak_burst, 4),
                      "launches": 4 * iters}
    return res


def _time_bwd(fa, device, stream, q, k, v, out, do, lse, dq, dk, dv, delta, causal, warmup, iters):
    """Mean ms of one fa_bwd call over `iters` back-to-back calls (CUDA events on `stream`)."""
    def call():
        fa.fa_bwd(q, k, v, out, do, lse, dq=dq, dk=dk, dv=dv, delta=delta, causal=causal, stream=stream)

    for _ in range(warmup):
        call()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        call()
    e1.record(stream)
    torch.cuda.synchronize(device)
    st, where = fa.fa_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} at {where} after the backward leg")
    return e0.elapsed_time(e1) / iters


def run_paged_leg(fa, device, stream, q, k_h, v_h, causal, flops, warmup, rank, iters=20):
    """fa_fwd_paged on the main workload with K/V scattered over shuffled page pools."""
    res = {"what": "the main workload with K/V in page pools (shuffled page order, block table), "
                   "fa_fwd_paged; TFLOPS and fraction of contiguous fa_fwd timed the same way",
           "launches_per_size": iters}
    out = torch.empty_like(q)
    k, v = k_h.to(device), v_h.to(device)

    def timed(call):
        for _ in range(warmup):
            call()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            call()
        e1.record(stream)
        torch.cuda.synchronize(device)
        return flops / (e0.elapsed_time(e1) / iters * 1e-3) / 1e12

    dense_tflops = timed(lambda: fa.fa_fwd(q, k, v, out=out, causal=causal, return_lse=False, stream=stream))
    res["contiguous_tflops"] = round(dense_tflops, 1)
    del k, v
    for ps in (16, 64, 256):
        kc, vc, table = fa_inputs.paged_kv(k_h, v_h, ps, seed=rank + 1, fill=0.0)
        kc, vc, table = kc.to(device), vc.to(device), table.to(device)
        tf = timed(lambda: fa.fa_fwd_paged(q, kc, vc, table, out=out, causal=causal, return_lse=False,
                                           stream=stream))
        res[f"page_{ps}"] = {"tflops": round(tf, 1), "frac_of_contiguous": round(tf / dense_tflops, 3)}
        del kc, vc, table
    return res


def run_varlen_leg(fa, device, stream, iters, warmup, ws):
    w = fa_inputs.WORKLOADS["varlen_bf16_32x64"]
    case = fa_inputs.workload_inputs("varlen_bf16_32x64")
    qp, kp, vp = case.q_pad.to(device), case.k_pad.to(device), case.v_pad.to(device)
    idx, cu = case.indices.to(device), case.cu_seqlens.to(device)
    H, D = w["H"], w["D"]
    qu = torch.empty((case.nnz, H, D), device=device, dtype=qp.dtype)
    ku, vu, ou = torch.empty_like(qu), torch.empty_like(qu), torch.empty_like(qu)
    lse = torch.empty((H, case.nnz), device=device, dtype=torch.float32)
    out_pad = torch.empty_like(qp)
    # L2 flush between timed calls (the inputs here are L2-sized): a reduction READS a 2x-L2
    # buffer, so L2 is left holding clean lines and no timed kernel pays for write-backs.
    flush = torch.ones(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    flush_out = torch.empty((), dtype=torch.int64, device=device)

    def flush_l2():
        torch.sum(flush, dim=0, dtype=torch.int64, out=flush_out)

    def call():
        fa.fa_unpad_qkv(qp, kp, vp, idx, outs=(qu, ku, vu), stream=stream)
        fa.fa_varlen_fwd(qu, ku, vu, cu, case.max_seqlen, out=ou, lse=lse, stream=stream)
        fa.fa_pad(ou, idx, 1, case.total_len, out=out_pad, stream=stream)

    for _ in range(max(warmup, 3)):
        call()
    torch.cuda.synchronize(device)
    n_ev = 6
    comp = [[], [], []]
    whole = []
    for it in range(iters):
        # keep the GPU busy while the host queues the whole call, so the events time the
        # kernels and not the host's launch gaps
        flush_l2()
        torch.cuda._sleep(400000)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
        ev[0].record(stream)
        fa.fa_unpad_qkv(qp, kp, vp, idx, outs=(qu, ku, vu), stream=stream)
        ev[1].record(stream)
        fa.fa_varlen_fwd(qu, ku, vu, cu, case.max_seqlen, out=ou, lse=lse, stream=stream)
        ev[2].record(stream)
        fa.fa_pad(ou, idx, 1, case.total_len, out=out_pad, stream=stream)
        ev[3].record(stream)
        torch.cuda.synchronize(device)
        whole.append(ev[0].elapsed_time(ev[3]) * 1e3)
        for c in range(3):
            comp[c].append(ev[c].elapsed_time(ev[c + 1]) * 1e3)
    # the same path as one launch (unpad and pad folded into the attention kernel)
    fused = []
    for it in range(iters):
        flush_l2()
        torch.cuda._sleep(400000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fa.fa_varlen_fwd_padded(qp, kp, vp, idx, cu, case.max_seqlen, out=out_pad, lse=lse, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        fused.append(e0.elapsed_time(e1) * 1e3)
    flops = 4.0 * H * D * sum(int(x) ** 2 for x in (case.cu_seqlens[1:] - case.cu_seqlens[:-1]))
    us = statistics.median(fused)
    us3 = statistics.median(whole)
    return {"value": round(us, 2), "unit": "us/call",
            "stat": f"median of {iters}, L2 flushed before each call by reading a 256 MiB buffer (no dirty "
                    f"lines left), launches queued ahead (GPU time)",
            "config": "32 seqs x 64 tokens, H=16 D=128 bf16, padded (1,4096,16,128), non-causal; "
                      "fa_varlen_fwd_padded (unpad + attention + pad in one launch)",
            "gpu_launches_per_call": 1,
            "three_launch_path": {"value": round(us3, 2), "unit": "us/call",
                                  "calls": "fa_unpad_qkv + fa_varlen_fwd + fa_pad",
                                  "components_us_median": {"unpad_qkv": round(statistics.median(comp[0]), 2),
                                                           "varlen_fwd": round(statistics.median(comp[1]), 2),
                                                           "pad_out": round(statistics.median(comp[2]), 2)},
                                  "components_note": "each from the event before its launch to the event after "
                                                     "it, so each includes the GPU's gap between the previous "
                                                     "kernel's end and its own start (about 2 us), which a "
                                                     "profiler's per-kernel duration leaves out",
                                  "varlen_fwd_tflops": round(flops / (statistics.median(comp[1]) * 1e-6) / 1e12, 2)}}


def run_padding_hbm_leg(fa, device, stream, iters):
    """unpad / pad GB/s on the packed structure scaled past L2: (1, 262144, 16, 128) bf16 = 1 GiB
    padded, half the positions valid. Algorithmic bytes: unpad reads and writes nnz rows plus the
    indices; pad reads nnz rows and the indices and writes every one of the total rows; unpad_qkv
    gathers the same rows from three distinct 1 GiB tensors in one launch."""
    _, peak_bw, peak_kind, _ = load_peaks()
    L, H, D = 262144, 16, 128
    nnz = L // 2
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    x = torch.randn((1, L, H, D), generator=g, dtype=torch.float32).to(torch.bfloat16).to(device)
    xk, xv = torch.empty_like(x).copy_(x), torch.empty_like(x).copy_(x)  # distinct buffers for the q, k, v gather
    idx = fa_inputs.valid_indices(L, nnz, seed=6).to(device)
    u = torch.empty((nnz, H, D), device=device, dtype=torch.bfloat16)
    uk, uv = torch.empty_like(u), torch.empty_like(u)
    out = torch.empty_like(x)
    row = H * D * 2
    res = {}
    for name, fn, nbytes in (
            ("unpad", lambda: fa.fa_unpad(x, idx, out=u, stream=stream), 2 * nnz * row + 8 * nnz),
            ("pad", lambda: fa.fa_pad(u, idx, 1, L, out=out, stream=stream), nnz * row + L * row + 8 * nnz),
            ("unpad_qkv", lambda: fa.fa_unpad_qkv(x, xk, xv, idx, outs=(u, uk, uv), stream=stream),
             3 * 2 * nnz * row + 8 * nnz)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(device)
        us = e0.elapsed_time(e1) / iters * 1e3
        gbs = nbytes / (us * 1e-6) / 1e9
        res[name] = {"us": round(us, 2), "bytes": nbytes, "achieved_gbs": round(gbs, 1), "peak_gbs": peak_bw,
                     "frac": round(gbs / peak_bw, 4), "peak_kind": f"{peak_kind} HBM copy"}
    res["config"] = ("(1, 262144, 16, 128) bf16 padded (1 GiB; three of them for unpad_qkv), 131072 valid rows; "
                     "inputs larger than L2")
    return res


# MUFU exp2 throughput of one SM per clock (sm_100, measured by a probe kernel: 16 results per
# clock for ex2.approx.f32 and for the packed f16x2 / bf16x2 forms alike).
MUFU_EXP2_PER_CLK_SM = 16
NUM_SMS = 148


def attention_exps(B: int, H: int, S: int, causal: bool) -> float:
    """One exp2 per visible score: S*S per (batch, head), S*(S+1)/2 when causal."""
    return float(B * H * (S * (S + 1) // 2 if causal else S * S))


def config_roofline(flops: float, exps: float, seconds: float, peak_tf: float, sm_mhz: float) -> dict:
    """Tensor time (FLOPs / peak) against exp time (exps / MUFU rate at the sampled clock): the
    larger is the bound; frac = that bound's time / the measured time."""
    t_mma = flops / (peak_tf * 1e12)
    t_exp = exps / (MUFU_EXP2_PER_CLK_SM * NUM_SMS * sm_mhz * 1e6)
    bound = "tensor" if t_mma >= t_exp else "exp (MUFU)"
    return {"bound": bound, "t_mma_us": round(t_mma * 1e6, 1), "t_exp_us": round(t_exp * 1e6, 1),
            "frac": round(max(t_mma, t_exp) / seconds, 4), "mufu_clock_mhz": round(sm_mhz, 0)}


def run_configs_leg(fa, device, stream, warmup, sm_mhz, main_ms, varlen):
    """Every workload of the pages on this GPU. Dense ones: fa_fwd, 20 launches after warm-up
    (the small fp16 case: 200 back-to-back calls, microseconds per call); inputs are larger
    than L2 except for the small case, whose point is the per-call latency."""
    peak_burst, peak_bw, _, _ = load_peaks()
    res = {}
    for name in ("dense_fp16_small", "vit_bf16", "llm_causal_bf16", "hdim_sweep_fp16_d32", "hdim_sweep_fp16_d64",
                 "hdim_sweep_fp16_d128", "hdim_sweep_fp16_d256"):
        w = fa_inputs.WORKLOADS[name]
        B, S, H, D, causal = w["B"], w["S"], w["H"], w["D"], w["causal"]
        flops = fa.attention_flops(B, H, S, S, D, causal)
        exps = attention_exps(B, H, S, causal)
        entry = {"shape": f"B{B} H{H} S{S} D{D} {w['dtype']}{' causal' if causal else ''}"}
        if name == "llm_causal_bf16":
            ms = main_ms  # the main timed region above
            entry["source"] = "main timed region"
        else:
            q, k, v = (t.to(device) for t in fa_inputs.dense_qkv(B, S, H, D, fa_inputs.DTYPES[w["dtype"]], seed=0))
            out = torch.empty_like(q)
            lse = torch.empty((B, H, S), device=device, dtype=torch.float32)
            n = 200 if name == "dense_fp16_small" else 20
            for _ in range(max(warmup, 3)):
                fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize(device)
            ms = e0.elapsed_time(e1) / n
            entry["launches"] = n
            if name == "dense_fp16_small":
                # The same n calls captured in one CUDA graph and replayed: the per-call time
                # without the host's launch path (what a caller replaying a graph sees).
                side = torch.cuda.Stream(device)
                side.wait_stream(torch.cuda.current_stream(device))
                with torch.cuda.stream(side):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=side):
                        for _ in range(n):
                            fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal)
                torch.cuda.current_stream(device).wait_stream(side)
                g.replay()
                torch.cuda.synchronize(device)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize(device)
                entry["graph_us_per_call"] = round(e0.elapsed_time(e1) / n * 1e3, 2)
                del g
            del q, k, v, out, lse
        entry["ms"] = round(ms, 4)
        entry["tflops"] = round(flops / (ms * 1e-3) / 1e12, 1)
        if name == "dense_fp16_small":
            entry["us_per_call"] = round(ms * 1e3, 2)
            entry["bound"] = "launch latency (8.4 MFLOP per call; the pages' small case)"
        else:
            entry.update(config_roofline(flops, exps, ms * 1e-3, peak_burst, sm_mhz))
        res[name] = entry
    v = varlen
    res["varlen_bf16_32x64"] = {"shape": "32 x 64 tokens, H16 D128 bf16, padded (1, 4096, 16, 128)",
                                "us_per_call": v["value"], "path": "fa_varlen_fwd_padded (one launch)",
                                "three_launch_us_per_call": v["three_launch_path"]["value"],
                                "bound": "latency (the inputs sit in L2); see varlen"}
    st, where = fa.fa_device_status(stream=stream)
    if st != 0:
        raise RuntimeError(f"device status {st} at {where} after the configs leg")
    return res


def run_all_configs(args):
    """TFLOPS of fa_fwd on every dense workload (informational; not the headline line)."""
    import tiled_exact_attention_fwd_b200 as fa
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peak_burst, _, _, _ = load_peaks()
    for name, w in fa_inputs.WORKLOADS.items():
        if w["kind"] != "dense":
            continue
        B, S, H, D, causal = w["B"], w["S"], w["H"], w["D"], w["causal"]
        q, k, v = (t.to(device) for t in fa_inputs.dense_qkv(B, S, H, D, fa_inputs.DTYPES[w["dtype"]], seed=0))
        out = torch.empty_like(q)
        lse = torch.empty((B, H, S), device=device, dtype=torch.float32)
        for _ in range(max(args.warmup, 3)):
            fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)
        torch.cuda.synchronize(device)
        n = max(1, min(args.steps, 50))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fa.fa_fwd(q, k, v, out=out, lse=lse, causal=causal, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / n
        tf = fa.attention_flops(B, H, S, S, D, causal) / (ms * 1e-3) / 1e12
        print(json.dumps({"workload": name, "us": round(ms * 1e3, 1), "tflops": round(tf, 1),
                          "frac_vs_burst": round(tf / peak_burst, 4), "launches": n}), flush=True)
        del q, k, v, out, lse


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    ws, rank, local = dist_info()
    if rank != 0:
        return
    import oracle
    w = fa_inputs.WORKLOADS[WORKLOAD]
    nth = oracle.max_threads()
    # Each step: the oracle on a bounded sample (whole heads, about 3 s of CPU work).
    per = []
    heads_used = flops_used = None
    for i in range(args.warmup + args.steps):
        tf, secs, nheads, fl, _ = oracle_sample(budget_s=3.0, max_heads=8)
        if i >= args.warmup:
            per.append((tf, secs))
            heads_used, flops_used = nheads, fl
    value = statistics.mean(t for t, _ in per)
    ms = statistics.mean(s for _, s in per) * 1e3
    sample = (f"all 8192 query rows of {heads_used} of the 32 heads of the causal S=8192 D=128 workload, "
              f"{flops_used:.3g} flops per step, float64 OpenMP")
    res = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1))", "impl": "reference",
           "config": {"workload": "causal attention fwd, B=1 H=32 S=8192 D=128 bf16, scale 1/sqrt(128)",
                      "B": w["B"], "H": w["H"], "S": w["S"], "D": w["D"], "causal": True},
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": nth, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def launch_local_ranks(n: int) -> int:
    """Runs this script again under torch.distributed.run with n local ranks (one per GPU, every
    rank on the same workload) and returns its exit code; rank 0 prints the JSON line."""
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def run_cpu_stub(args):
    """The N-rank plumbing without a GPU: CPU ranks over gloo, each step a small CPU matmul,
    the time the max over ranks. A test of the launcher and the rank logic, not a measurement."""
    import datetime

    import torch.distributed as dist
    ws, rank, _ = dist_info()
    if ws > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    a = torch.randn(128, 128)
    for _ in range(args.warmup):
        a @ a
    if ws > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        a @ a
    ms = max_over_ranks((time.perf_counter() - t0) / args.steps * 1e3, ws, torch.device("cpu"))
    if ws > 1:
        dist.barrier()
    if rank == 0:
        print(json.dumps({"metric": METRIC, "value": None, "unit": "TFLOPS", "n_gpus": ws, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": round(ms, 4), "scaling": "weak",
                          "stub": "CPU ranks over gloo: a test of the launcher, not a measurement"}), flush=True)
    if ws > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only-main", action="store_true", help="time the main kernel only (for profiling)")
    ap.add_argument("--only-padding", action="store_true", help="run the unpad/pad HBM leg only (for profiling)")
    ap.add_argument("--only-backward", action="store_true", help="run the backward leg only (for profiling)")
    ap.add_argument("--all-configs", action="store_true",
                    help="print one informational line per workload (dense/causal/head-dim sweep)")
    ap.add_argument("--cpu-stub", action="store_true", help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # N GPUs of this node: one process per GPU under torch.distributed.run
        sys.exit(launch_local_ranks(args.gpus))
    if args.cpu_stub:
        run_cpu_stub(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.all_configs:
        run_all_configs(args)
    elif args.only_backward:
        import tiled_exact_attention_fwd_b200 as fa
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        w = fa_inputs.WORKLOADS[WORKLOAD]
        B, S, H, D, causal = w["B"], w["S"], w["H"], w["D"], w["causal"]
        q, k, v = (t.to(device) for t in fa_inputs.dense_qkv(B, S, H, D, fa_inputs.DTYPES[w["dtype"]], seed=0))
        out = torch.empty_like(q)
        lse = torch.empty((B, H, S), device=device, dtype=torch.float32)
        print(json.dumps(run_backward_leg(fa, device, torch.cuda.current_stream(device), q, k, v, out, lse, causal,
                                          args.warmup, 0, iters=max(args.steps, 1))))
    elif args.only_padding:
        import tiled_exact_attention_fwd_b200 as fa
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        print(json.dumps(run_padding_hbm_leg(fa, device, torch.cuda.current_stream(device), max(args.steps, 1))))
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
