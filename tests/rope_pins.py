"""Checks that pin the 3D RoPE oracle to facts other than itself.

Each check takes `rope`, a function with the signature of
oracle.rope_ref.rope3d_ref, and raises AssertionError on failure. The facts
are those any rotary embedding has, plus the layout the reading fixes
(recorded with the oracle: contiguous t, h, w sections of the head dimension,
adjacent pairs, frequencies 1 down to base^(-(D_a - 2) / D_a) per section):

  identity     the token at position (0, 0, 0) is unchanged.
  norm         every token keeps its Euclidean norm (rotations).
  linear       rope(a x + b y) = a rope(x) + b rope(y).
  relative     <rope(q) at p, rope(k) at p'> depends only on p - p', per axis
               (the property rotary embedding exists for).
  compose      rotating by frame a, then by frame b, equals rotating by a + b.
  sections     moving a token along t, h or w changes only that axis's dims:
               t dims [0, D_t), h dims [D_t, D_t + D_h), w dims after; h is
               the grid row (r // W), w the column (r % W).
  pairs        a vector on one dim stays within its adjacent pair (2i, 2i+1).
  unit_pair    the first pair of each section turns by exactly the position,
               in radians, counter-clockwise: (1, 0) -> (cos p, sin p).
  schedule     the pair frequencies of a section fall geometrically from 1 to
               base^(-(D_a - 2) / D_a), base 10000 (the standard schedule).
"""
from __future__ import annotations

import math

import numpy as np


def _tok(D, rng, n=1):
    return rng.standard_normal((n, D))


def check_identity(rope, D=64):
    rng = np.random.default_rng(41)
    x = rng.standard_normal((1, 1, D))
    y = rope(x, grid_w=7, t0=0)
    assert np.allclose(y, x, rtol=0, atol=1e-15), "position (0,0,0) must be the identity"


def check_norm(rope, D=64, T=3, S=12, W=4):
    rng = np.random.default_rng(42)
    x = rng.standard_normal((T, S, D))
    y = rope(x, grid_w=W, t0=17)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13, atol=0)


def check_linear(rope, D=32, T=2, S=6, W=3):
    rng = np.random.default_rng(43)
    x, y = rng.standard_normal((2, T, S, D))
    a, b = 0.7, -1.3
    assert np.allclose(rope(a * x + b * y, grid_w=W, t0=5), a * rope(x, grid_w=W, t0=5) +
                       b * rope(y, grid_w=W, t0=5), rtol=1e-13, atol=1e-13)


def _at(rope, v, t, h, w, W, D):
    """rope of vector v placed at frame t, grid (h, w)."""
    S = h * W + w + 1
    x = np.zeros((1, S, D))
    x[0, h * W + w] = v
    return rope(x, grid_w=W, t0=t)[0, h * W + w]


def check_relative(rope, D=64, W=9):
    rng = np.random.default_rng(44)
    q, k = rng.standard_normal((2, D))
    for (t, h, w), (t2, h2, w2) in (((3, 1, 2), (1, 0, 5)), ((10, 4, 0), (2, 2, 8))):
        d0 = _at(rope, q, t, h, w, W, D) @ _at(rope, k, t2, h2, w2, W, D)
        for sh in ((5, 0, 0), (0, 3, 0), (0, 0, 1), (40, 2, 0)):
            d1 = (_at(rope, q, t + sh[0], h + sh[1], w + sh[2], W + 2, D) @
                  _at(rope, k, t2 + sh[0], h2 + sh[1], w2 + sh[2], W + 2, D))
            assert abs(d1 - d0) < 1e-11 * (1 + abs(d0)), ("relative", sh, d0, d1)


def check_compose(rope, D=64):
    rng = np.random.default_rng(45)
    x = rng.standard_normal((1, 1, D))                 # token 0: h = w = 0
    for a, b in ((1, 2), (7, 30), (0, 5)):
        assert np.allclose(rope(rope(x, grid_w=3, t0=a), grid_w=3, t0=b),
                           rope(x, grid_w=3, t0=a + b), rtol=1e-12, atol=1e-12), ("compose", a, b)


def _sections(D):
    dh = 2 * (D // 6)
    return D - 2 * dh, dh, dh


def check_sections(rope, W=5):
    rng = np.random.default_rng(46)
    for D in (64, 128, 32):
        Dt, Dh, Dw = _sections(D)
        v = rng.standard_normal(D)
        base = _at(rope, v, 0, 0, 0, W, D)
        moved = {"t": _at(rope, v, 1, 0, 0, W, D), "h": _at(rope, v, 0, 1, 0, W, D),
                 "w": _at(rope, v, 0, 0, 1, W, D)}
        spans = {"t": (0, Dt), "h": (Dt, Dt + Dh), "w": (Dt + Dh, D)}
        for axis, y in moved.items():
            lo, hi = spans[axis]
            changed = np.nonzero(np.abs(y - base) > 1e-12)[0]
            assert changed.size and changed.min() >= lo and changed.max() < hi, (D, axis, changed)


def check_pairs(rope, D=64):
    for d in (0, 1, 5, 24, 45, 63):
        v = np.zeros(D)
        v[d] = 1.0
        y = _at(rope, v, 3, 2, 4, 6, D)
        pair = {d - d % 2, d - d % 2 + 1}
        assert set(np.nonzero(np.abs(y) > 1e-15)[0]) <= pair, ("pairs", d)


def check_unit_pair(rope, D=64):
    Dt, Dh, Dw = _sections(D)
    for first, pos in ((0, (2.0, 0, 0)), (Dt, (0, 3.0, 0)), (Dt + Dh, (0, 0, 5.0))):
        v = np.zeros(D)
        v[first] = 1.0
        p = max(pos)
        y = _at(rope, v, int(pos[0]), int(pos[1]), int(pos[2]), 8, D)
        assert abs(y[first] - math.cos(p)) < 1e-14 and abs(y[first + 1] - math.sin(p)) < 1e-14, first


def check_schedule(rope, D=64, base=10000.0):
    Dt, Dh, Dw = _sections(D)
    for start, size, pos in ((0, Dt, (1, 0, 0)), (Dt, Dh, (0, 1, 0)), (Dt + Dh, Dw, (0, 0, 1))):
        for i in range(size // 2):
            v = np.zeros(D)
            v[start + 2 * i] = 1.0
            y = _at(rope, v, pos[0], pos[1], pos[2], 4, D)
            ang = math.atan2(y[start + 2 * i + 1], y[start + 2 * i])
            assert abs(ang - base ** (-2.0 * i / size)) < 1e-13, (start, i, ang)


ALL = {
    "identity": check_identity,
    "norm": check_norm,
    "linear": check_linear,
    "relative": check_relative,
    "compose": check_compose,
    "sections": check_sections,
    "pairs": check_pairs,
    "unit_pair": check_unit_pair,
    "schedule": check_schedule,
}
