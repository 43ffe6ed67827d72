"""Helpers for the GPU tests: seeded inputs on the device, oracle comparison."""
from __future__ import annotations

import numpy as np
import torch

from frame_wise_gated_scan_b200 import inputs
from oracle import gdn_scan_ref, rel_frobenius

TOL_F32 = 1e-5     # relative Frobenius error per frame, fp32-input path
TOL_BF16 = 2e-2    # relative Frobenius error per frame, bf16-input path


def device_workload(wl: inputs.Workload, T: int | None = None, device="cuda"):
    """q, k, v (bf16 or fp32), gamma, beta (fp32) on the device, head by head."""
    T = wl.T if T is None else T
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    shape = (wl.B, wl.H, T, wl.S, wl.D)
    q = torch.empty(shape, dtype=dt, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    g = torch.empty((wl.B, wl.H, T), dtype=torch.float32, device=device)
    be = torch.empty_like(g)
    for b, h, qq, kk, vv, gg, bb in inputs.iter_heads_packed(wl, T):
        if wl.dtype == "bf16":
            for dst, src in ((q, qq), (k, kk), (v, vv)):
                dst[b, h].copy_(torch.from_numpy(src.view(np.int16)).view(torch.bfloat16))
        else:
            for dst, src in ((q, qq), (k, kk), (v, vv)):
                dst[b, h].copy_(torch.from_numpy(src))
        g[b, h].copy_(torch.from_numpy(gg))
        be[b, h].copy_(torch.from_numpy(bb))
    return q, k, v, g, be


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_head(wl: inputs.Workload, b: int, h: int, T: int | None = None, state_in=None,
                delta: bool = True):
    q, k, v, g, be = inputs.head(wl, b, h, T)
    return gdn_scan_ref(q, k, v, g, be, state_in=state_in, delta=delta)


def assert_close(out, ref_out, state, ref_state, tol, what=""):
    out = np.asarray(out, np.float64)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    e_out = rel_frobenius(out, ref_out)            # per leading index (frame)
    worst = float(np.max(e_out))
    assert worst <= tol, f"{what}: worst per-frame rel. Frobenius error {worst:.3e} > {tol}"
    if state is not None:
        state = np.asarray(state, np.float64)
        assert np.all(np.isfinite(state)), f"{what}: non-finite state"
        e_st = float(np.max(rel_frobenius(state, ref_state)))
        assert e_st <= tol, f"{what}: state rel. Frobenius error {e_st:.3e} > {tol}"
        return worst, e_st
    return worst, None
