"""Seeded synthetic inputs for the frame-wise Gated DeltaNet scan.

This module only draws and packs numbers: it holds none of the recurrence's
arithmetic, so both the float64 oracle and the CUDA path can be fed from it.

Workloads (the shapes of the SANA-WM setting: 961 latent frames for a 60 s
720p clip, as stated in "NVIDIA Apresenta SANA-WM ..." (acheiumaia.com.br),
section "1. Atenção Linear Híbrida com Gated DeltaNet (GDN)"; S = 22x40 or
30x45 spatial tokens per latent frame):

  tiny     B=1 H=2  D=32  T=8   S=64    fp32  Q,K,V ~ N(0,1); gamma ~ U(.85,1); beta ~ U(0,1)
  short    B=1 H=16 D=64  T=21  S=880   bf16  Q,K,V ~ N(0,1); gamma = sigmoid(N(3,.5)); beta = sigmoid(N(0,1))
  rollout  B=1 H=32 D=64  T=961 S=880   bf16  Q,V ~ N(0,1); K rows L2-normalised; gamma ~ U(.95,1); beta ~ U(.2,1)
  step     the rollout tensors, fed one frame per call
  stress   B=4 H=16 D=128 T=241 S=1350  bf16  K rows = unit direction * exp(N(0,1)); gamma ~ U(.99,1); beta = 1

Every frame of every head has its own generator, seeded with
(config seed, b, h, t), so any frame can be regenerated on its own. Inside a
frame the draws come in the order Q, K (then the log-norms for "stress"), V,
gamma, beta. Samples are float32; bf16 workloads round Q, K, V to bf16 with
round-to-nearest-even, and both sides consume the rounded values.
"""
from __future__ import annotations

import dataclasses
import math
import os

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    T: int
    S: int
    dtype: str          # "f32" or "bf16": the element type of q, k, v and out
    seed: int
    key_mode: str       # "gauss", "l2" or "lognormal"
    gate_mode: str      # see _draw_gates

    @property
    def heads(self) -> int:
        return self.B * self.H

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 32, 8, 64, "f32", 1, "gauss", "tiny"),
    "short": Workload("short", 1, 16, 64, 21, 880, "bf16", 2, "gauss", "short"),
    "rollout": Workload("rollout", 1, 32, 64, 961, 880, "bf16", 3, "l2", "rollout"),
    "step": Workload("step", 1, 32, 64, 961, 880, "bf16", 3, "l2", "rollout"),
    "stress": Workload("stress", 4, 16, 128, 241, 1350, "bf16", 5, "lognormal", "stress"),
}


def _rng(seed: int, b: int, h: int, t: int) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(np.random.SeedSequence([seed, b, h, t])))


def _sigmoid(x: float) -> float:
    return 1.0 / (1.0 + math.exp(-x))


def _draw_gates(rng: np.random.Generator, mode: str) -> tuple[float, float]:
    if mode == "tiny":
        return float(np.float32(rng.uniform(0.85, 1.0))), float(np.float32(rng.uniform(0.0, 1.0)))
    if mode == "short":
        g = _sigmoid(rng.normal(3.0, 0.5))
        b = _sigmoid(rng.normal(0.0, 1.0))
        return float(np.float32(g)), float(np.float32(b))
    if mode == "rollout":
        return float(np.float32(rng.uniform(0.95, 1.0))), float(np.float32(rng.uniform(0.2, 1.0)))
    if mode == "stress":
        return float(np.float32(rng.uniform(0.99, 1.0))), 1.0
    raise ValueError(mode)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def frame(wl: Workload, b: int, h: int, t: int, S: int | None = None):
    """One frame of one head: (q, k, v) as float32 [S, D] holding exactly
    representable values of the workload's dtype, and (gamma, beta) floats."""
    S = wl.S if S is None else S
    rng = _rng(wl.seed, b, h, t)
    q = rng.standard_normal((S, wl.D), dtype=np.float32)
    k = rng.standard_normal((S, wl.D), dtype=np.float32)
    if wl.key_mode in ("l2", "lognormal"):
        k = k / np.sqrt(np.sum(k * k, axis=1, keepdims=True, dtype=np.float32))
    if wl.key_mode == "lognormal":
        z = rng.standard_normal((S,), dtype=np.float32)
        k = k * np.exp(z)[:, None]
    v = rng.standard_normal((S, wl.D), dtype=np.float32)
    gamma, beta = _draw_gates(rng, wl.gate_mode)
    if wl.dtype == "bf16":
        q, k, v = (bf16_to_f32(bf16_round(a)) for a in (q, k, v))
    return q.astype(np.float32), k.astype(np.float32), v.astype(np.float32), gamma, beta


def head(wl: Workload, b: int, h: int, T: int | None = None):
    """All frames of one head: q, k, v float32 [T, S, D]; gamma, beta float32 [T]."""
    T = wl.T if T is None else T
    q = np.empty((T, wl.S, wl.D), np.float32)
    k = np.empty_like(q)
    v = np.empty_like(q)
    g = np.empty((T,), np.float32)
    be = np.empty((T,), np.float32)
    for t in range(T):
        q[t], k[t], v[t], g[t], be[t] = frame(wl, b, h, t)
    return q, k, v, g, be


def _head_packed(args):
    wl, b, h, T = args
    q, k, v, g, be = head(wl, b, h, T)
    if wl.dtype == "bf16":
        q, k, v = bf16_round(q), bf16_round(k), bf16_round(v)
    return b, h, q, k, v, g, be


def iter_heads_packed(wl: Workload, T: int | None = None, processes: int | None = None):
    """Yield (b, h, q, k, v, gamma, beta) per head, with q/k/v already in the
    workload's storage type (uint16 bf16 bit patterns or float32). Large
    workloads are drawn by a spawn-started process pool."""
    T = wl.T if T is None else T
    jobs = [(wl, b, h, T) for b in range(wl.B) for h in range(wl.H)]
    work = wl.heads * T * wl.S * wl.D
    if processes is None:
        processes = min(len(jobs), os.cpu_count() or 1, 32) if work > (1 << 24) else 1
    if processes <= 1:
        for j in jobs:
            yield _head_packed(j)
        return
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    with ctx.Pool(processes) as pool:
        for item in pool.imap(_head_packed, jobs):
            yield item


def full(wl: Workload, T: int | None = None):
    """Whole workload as float32 arrays q, k, v [B,H,T,S,D], gamma, beta [B,H,T].
    Meant for small workloads (the oracle side)."""
    T = wl.T if T is None else T
    q = np.empty((wl.B, wl.H, T, wl.S, wl.D), np.float32)
    k = np.empty_like(q)
    v = np.empty_like(q)
    g = np.empty((wl.B, wl.H, T), np.float32)
    be = np.empty_like(g)
    for b in range(wl.B):
        for h in range(wl.H):
            q[b, h], k[b, h], v[b, h], g[b, h], be[b, h] = head(wl, b, h, T)
    return q, k, v, g, be


def state(wl: Workload, seed_offset: int = 1000, scale: float = 1.0):
    """A seeded non-zero initial state M_0 [B,H,D,D] (float32), for tests that
    carry a state into a call."""
    out = np.empty((wl.B, wl.H, wl.D, wl.D), np.float32)
    for b in range(wl.B):
        for h in range(wl.H):
            r = _rng(wl.seed + seed_offset, b, h, 0)
            out[b, h] = scale * r.standard_normal((wl.D, wl.D), dtype=np.float32) / math.sqrt(wl.D)
    return out


def algorithmic_bytes(wl: Workload, T: int | None = None) -> int:
    """Bytes one scan must move at least: q, k, v read and out written once,
    gamma and beta read, the state written once."""
    T = wl.T if T is None else T
    n = wl.heads * T * wl.S * wl.D
    return 4 * n * wl.elt_bytes + wl.heads * T * 8 + wl.heads * wl.D * wl.D * 4


def flops(wl: Workload, T: int | None = None) -> int:
    """Floating-point operations of the three S-by-D-by-D contractions per frame and head."""
    T = wl.T if T is None else T
    return 6 * wl.heads * T * wl.S * wl.D * wl.D


# ---- the causal temporal convolution (the companion of the GDN state in
# chunk-causal rollout): x [B][T][S][C] bf16, taps w [C][3] and bias [C] fp32,
# a carried last-frame cache [B][S][C] bf16.

@dataclasses.dataclass(frozen=True)
class ConvWorkload:
    name: str
    B: int
    T: int
    S: int
    C: int
    F: int        # frames per block
    seed: int

    def with_(self, **kw) -> "ConvWorkload":
        return dataclasses.replace(self, **kw)


# The rollout's shapes: 961 latent frames of 22 x 40 tokens, C = 2048 channels
# (32 heads x 64, the width of the GDN layer), blocks of 8 frames.
CONV_WORKLOADS = {
    "conv_rollout": ConvWorkload("conv_rollout", 1, 961, 880, 2048, 8, 7),
}


def conv_frame(wl: ConvWorkload, b: int, t: int) -> np.ndarray:
    """Frame t of sequence b: float32 [S, C] holding bf16 values, N(0, 1)."""
    rng = _rng(wl.seed, b, t, 0)
    return bf16_to_f32(bf16_round(rng.standard_normal((wl.S, wl.C), dtype=np.float32)))


def conv_params(wl: ConvWorkload):
    """Taps w [C, 3] ~ N(0, 1/3) and bias [C] ~ N(0, 0.01), float32."""
    rng = _rng(wl.seed + 2000, 0, 0, 0)
    w = (rng.standard_normal((wl.C, 3), dtype=np.float32) / np.float32(math.sqrt(3.0)))
    bias = rng.standard_normal((wl.C,), dtype=np.float32) * np.float32(0.1)
    return w.astype(np.float32), bias.astype(np.float32)


def conv_cache(wl: ConvWorkload) -> np.ndarray:
    """A carried cache [B, S, C]: float32 holding bf16 values, N(0, 1)."""
    out = np.empty((wl.B, wl.S, wl.C), np.float32)
    for b in range(wl.B):
        rng = _rng(wl.seed + 1000, b, 0, 0)
        out[b] = bf16_to_f32(bf16_round(rng.standard_normal((wl.S, wl.C), dtype=np.float32)))
    return out


def conv_full(wl: ConvWorkload) -> np.ndarray:
    """Whole input x [B, T, S, C] float32 (small workloads)."""
    x = np.empty((wl.B, wl.T, wl.S, wl.C), np.float32)
    for b in range(wl.B):
        for t in range(wl.T):
            x[b, t] = conv_frame(wl, b, t)
    return x


def conv_bytes(wl: ConvWorkload) -> int:
    """Bytes one call must move: x read and y written once (bf16), the taps
    and bias, the cache read and written."""
    n = wl.B * wl.T * wl.S * wl.C
    return 2 * n * 2 + wl.C * 16 + 2 * wl.B * wl.S * wl.C * 2


# ---- device-side draws for timing runs. Seeded and with the workloads'
# distributions, but a different stream from the per-frame generators above:
# the parity tests use those; only the benchmark uses these (kernel time does
# not depend on the values).

def device_draw(wl: Workload, device, seed_offset: int = 0):
    """q, k, v [B,H,T,S,D] (bf16 or fp32) and gamma, beta [B,H,T] fp32 drawn
    on `device` with torch's generator, following the workload's recipe."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_003 * wl.seed + seed_offset)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    shape = (wl.B, wl.H, wl.T, wl.S, wl.D)

    def normal(*shp):
        return torch.randn(shp, generator=gen, device=device, dtype=torch.float32)

    def uniform(lo, hi, shp):
        return lo + (hi - lo) * torch.rand(shp, generator=gen, device=device, dtype=torch.float32)

    q = normal(*shape).to(dt)
    k = normal(*shape)
    if wl.key_mode in ("l2", "lognormal"):
        k = k / k.norm(dim=-1, keepdim=True)
    if wl.key_mode == "lognormal":
        k = k * torch.exp(normal(*shape[:-1], 1))
    k = k.to(dt)
    v = normal(*shape).to(dt)
    gs = (wl.B, wl.H, wl.T)
    if wl.gate_mode == "tiny":
        g, b = uniform(0.85, 1.0, gs), uniform(0.0, 1.0, gs)
    elif wl.gate_mode == "short":
        g, b = torch.sigmoid(3.0 + 0.5 * normal(*gs)), torch.sigmoid(normal(*gs))
    elif wl.gate_mode == "rollout":
        g, b = uniform(0.95, 1.0, gs), uniform(0.2, 1.0, gs)
    elif wl.gate_mode == "stress":
        g, b = uniform(0.99, 1.0, gs), torch.ones(gs, device=device)
    else:
        raise ValueError(wl.gate_mode)
    return q, k, v, g.contiguous(), b.contiguous()


def conv_device_draw(wl: ConvWorkload, device):
    """x [B,T,S,C] bf16, taps w [C,3], bias [C] fp32 and a cache [B,S,C] bf16,
    drawn on `device` with torch's generator (same distributions as above)."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(1_000_003 * wl.seed)
    x = torch.randn((wl.B, wl.T, wl.S, wl.C), generator=gen, device=device).to(torch.bfloat16)
    w = torch.randn((wl.C, 3), generator=gen, device=device) / math.sqrt(3.0)
    bias = 0.1 * torch.randn((wl.C,), generator=gen, device=device)
    cache = torch.randn((wl.B, wl.S, wl.C), generator=gen, device=device).to(torch.bfloat16)
    return x, w, bias, cache
