"""Float64 CPU oracle for 3D rotary position embedding (RoPE) of queries and keys.

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the CPU-baseline leg of the benchmark may import or run it. It
shares no code with the CUDA path.

Where it comes from
-------------------
The SANA-Video ICLR 2026 oral transcript (shadowingenglish.com), the part on
temporal modelling: the model adds 3D RoPE to its linear attention (and
temporal convolutions), applied to queries and keys before attention. The
talk gives no frequency layout, so the reading taken here is the plainest
extension of one-dimensional rotary embedding to the three axes of a latent
video (frame t, row h, column w of the token grid):

  * the head dimension D is cut into three contiguous sections, for t, h and
    w, of D_h = D_w = 2 * floor(D / 6) dims each and D_t = D - D_h - D_w
    (D = 64: 24 + 20 + 20; D = 128: 44 + 42 + 42);
  * inside a section of D_a dims, dims (2i, 2i + 1) form pair i
    (i < D_a / 2), rotated by the angle p_a * base^(-2i / D_a), base = 10000,
    where p_a is the token's position on that axis:
        (x, y) -> (x cos a - y sin a, x sin a + y cos a);
  * token r of frame t sits at h = r // W, w = r % W on a grid W tokens wide
    (22 x 40 for S = 880); t is the frame's absolute index in the video.

Everything runs in float64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["rope_sections", "rope_angles", "rope3d_ref"]


def rope_sections(D: int):
    """(D_t, D_h, D_w) for head dimension D."""
    if D % 2:
        raise ValueError("D must be even")
    dh = 2 * (D // 6)
    return D - 2 * dh, dh, dh


def rope_angles(D: int, t, h, w, base: float = 10000.0) -> np.ndarray:
    """Rotation angle of every pair for positions (t, h, w): [..., D // 2]."""
    t, h, w = (np.asarray(a, dtype=np.float64) for a in (t, h, w))
    out = []
    for pos, size in zip((t, h, w), rope_sections(D)):
        i = np.arange(size // 2, dtype=np.float64)
        freq = base ** (-2.0 * i / size)
        out.append(pos[..., None] * freq)
    return np.concatenate(out, axis=-1)


def rope3d_ref(x, grid_w: int, t0: int = 0, base: float = 10000.0):
    """Rotate x [..., T, S, D] (queries or keys of T frames of S tokens each):
    frame index t0 + tau for the tau-th frame, grid position (r // grid_w,
    r % grid_w) for token r. Returns float64 of the same shape."""
    x = np.asarray(x, dtype=np.float64)
    *lead, T, S, D = x.shape
    tau = np.arange(T, dtype=np.float64)[:, None] + t0
    r = np.arange(S)
    ang = rope_angles(D, np.broadcast_to(tau, (T, S)),
                      np.broadcast_to((r // grid_w)[None, :], (T, S)),
                      np.broadcast_to((r % grid_w)[None, :], (T, S)), base)     # [T, S, D/2]
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out
