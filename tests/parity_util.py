"""Comparison helpers for the GPU-vs-oracle parity tests (no attention arithmetic here).

Tolerances (stated once, used by every parity test):
  O    max |gpu - oracle| <= 2e-2 for bf16, 5e-3 for fp16;
  LSE  |gpu - oracle| <= 1e-3 * max(1, |oracle|) (relative 1e-3, absolute near zero);
  unpad / pad: bit-exact.
"""
import numpy as np
import torch

O_TOL = {torch.bfloat16: 2e-2, torch.float16: 5e-3}
LSE_REL = 1e-3


def assert_o_close(gpu_o, ref_o, dtype, what=""):
    g = gpu_o.detach().float().cpu().double().numpy() if isinstance(gpu_o, torch.Tensor) else np.asarray(gpu_o)
    r = np.asarray(ref_o, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - r)
    tol = O_TOL[dtype]
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"{what}: max |O - oracle| = {worst:.3g} > {tol} at {np.unravel_index(err.argmax(), err.shape)}"
    return worst


def assert_lse_close(gpu_lse, ref_lse, what=""):
    g = gpu_lse.detach().cpu().double().numpy() if isinstance(gpu_lse, torch.Tensor) else np.asarray(gpu_lse)
    r = np.asarray(ref_lse, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r) / np.maximum(1.0, np.abs(r))
    worst = float(err.max()) if err.size else 0.0
    assert worst <= LSE_REL, f"{what}: LSE rel err {worst:.3g} > {LSE_REL} at {np.unravel_index(err.argmax(), err.shape)}"
    return worst


def edge_rows(S, tile=128):
    """Row positions that sit on tile edges and at both ends."""
    rows = {0, 1, S - 1, S - 2}
    for t in range(tile, S, tile):
        rows |= {t - 1, t, t + 1}
    return sorted(r for r in rows if 0 <= r < S)
