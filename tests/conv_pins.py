"""Checks that pin the temporal-convolution oracle to facts other than itself.

Each check takes `conv`, a function with the signature of
oracle.conv_ref.temporal_conv_ref, and raises AssertionError on failure. The
facts (SANA-Video ICLR 2026 oral transcript, the part on the causal FFN with
temporal convolution; three centred taps is the reading recorded with the
oracle):

  correlate    one block with a zero (or given) cache equals numpy's
               correlate of the frame sequence padded with the cache in front
               and one zero frame behind: a library routine, not the oracle's
               loop.
  impulse      a single non-zero frame tau reaches frame tau+1 through the
               first tap, frame tau through the middle one, and frame tau-1
               through the last one, except when tau opens a block (the zero
               token separates the blocks): brute force on a tiny input.
  toeplitz     the whole call is one T x T matrix per channel, block-
               triangular above the diagonal: w0 on the sub-diagonal, w1 on the
               diagonal, w2 on the super-diagonal except at block ends.
  causal       a block's outputs do not change when later blocks change
               (block one cannot foresee block two), and do change with the
               previous block's last frame (block two sees block one's token).
  split        a call split at a block boundary, carrying the cache, equals one
               call; a split inside a block does not (the split adds a pad).
  one_frame    one frame per block is a two-tap causal filter: the last tap
               never contributes.
  cache_out    the cache handed on is exactly the last frame.
"""
from __future__ import annotations

import numpy as np


def _rel(x, y):
    d = float(np.linalg.norm(np.asarray(x) - np.asarray(y)))
    n = float(np.linalg.norm(np.asarray(y)))
    return d / max(n, 1e-300)


def _case(rng, T, S=3, C=4):
    x = rng.standard_normal((T, S, C))
    w = rng.standard_normal((C, 3))
    b = rng.standard_normal(C)
    return x, w, b


def check_correlate(conv, seed=31, T=7, S=3, C=4):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    cache = rng.standard_normal((S, C))
    for cin in (None, cache):
        y, _ = conv(x, w, b, cache=cin, frames_per_block=None)
        front = np.zeros((S, C)) if cin is None else cin
        for s in range(S):
            for c in range(C):
                a = np.concatenate([[front[s, c]], x[:, s, c], [0.0]])
                ref = np.correlate(a, w[c], mode="valid") + b[c]
                assert _rel(y[:, s, c], ref) < 1e-14, ("correlate", s, c)


def check_impulse(conv, seed=32, T=9, F=3, S=2, C=3):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((C, 3))
    amp = rng.standard_normal((S, C))
    for tau in range(T):
        x = np.zeros((T, S, C))
        x[tau] = amp
        y, _ = conv(x, w, None, cache=None, frames_per_block=F)
        expect = np.zeros((T, S, C))
        expect[tau] = w[:, 1] * amp
        if tau + 1 < T:
            expect[tau + 1] = w[:, 0] * amp                 # seen as the previous frame,
        if tau >= 1 and tau % F != 0:                       # across a block boundary too
            expect[tau - 1] = w[:, 2] * amp                 # seen as the next frame,
        assert np.array_equal(y, expect), ("impulse", tau)   # only inside a block


def check_toeplitz(conv, seed=33, T=10, F=4, S=2, C=3):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    cache = rng.standard_normal((S, C))
    y, _ = conv(x, w, b, cache=cache, frames_per_block=F)
    for c in range(C):
        A = np.zeros((T, T))
        for t in range(T):
            A[t, t] = w[c, 1]
            if t >= 1:
                A[t, t - 1] = w[c, 0]
            if t + 1 < T and (t + 1) % F != 0:
                A[t, t + 1] = w[c, 2]
        for s in range(S):
            ref = A @ x[:, s, c] + b[c]
            ref[0] += w[c, 0] * cache[s, c]
            assert _rel(y[:, s, c], ref) < 1e-14, ("toeplitz", c, s)


def check_causal(conv, seed=34, T=9, F=3, S=2, C=3):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    y, _ = conv(x, w, b, frames_per_block=F)
    for blk in range(T // F - 1):
        end = (blk + 1) * F
        x2 = x.copy()
        x2[end:] = rng.standard_normal(x2[end:].shape)       # rewrite every later block
        y2, _ = conv(x2, w, b, frames_per_block=F)
        assert np.array_equal(y2[:end], y[:end]), ("causal: saw a later block", blk)
        x3 = x.copy()
        x3[end - 1] += 1.0                                   # this block's last frame
        y3, _ = conv(x3, w, b, frames_per_block=F)
        assert not np.allclose(y3[end], y[end]), ("causal: next block misses the cached frame", blk)


def check_split(conv, seed=35, T=12, F=4, S=3, C=2):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    cache = rng.standard_normal((S, C))
    y, c_out = conv(x, w, b, cache=cache, frames_per_block=F)
    for cut in (F, 2 * F):
        y1, c1 = conv(x[:cut], w, b, cache=cache, frames_per_block=F)
        y2, c2 = conv(x[cut:], w, b, cache=c1, frames_per_block=F)
        assert np.array_equal(np.concatenate([y1, y2]), y), ("split", cut)
        assert np.array_equal(c2, c_out)
    y1, c1 = conv(x[:F + 1], w, b, cache=cache, frames_per_block=F)
    assert not np.allclose(y1[F], y[F]), "split inside a block must pad its last frame"


def check_one_frame(conv, seed=36, T=6, S=2, C=3):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    y, _ = conv(x, w, b, frames_per_block=1)
    w2 = w.copy()
    w2[:, 2] = rng.standard_normal(C)
    y2, _ = conv(x, w2, b, frames_per_block=1)
    assert np.array_equal(y, y2), "one frame per block: the next-frame tap contributed"
    for t in range(T):
        prev = x[t - 1] if t else 0.0
        assert _rel(y[t], w[:, 0] * prev + w[:, 1] * x[t] + b) < 1e-15


def check_cache_out(conv, seed=37, T=5, S=3, C=2):
    rng = np.random.default_rng(seed)
    x, w, b = _case(rng, T, S, C)
    for F in (1, 2, T):
        _, c = conv(x, w, b, frames_per_block=F)
        assert np.array_equal(c, x[T - 1])


ALL = {
    "correlate": check_correlate,
    "impulse": check_impulse,
    "toeplitz": check_toeplitz,
    "causal": check_causal,
    "split": check_split,
    "one_frame": check_one_frame,
    "cache_out": check_cache_out,
}
