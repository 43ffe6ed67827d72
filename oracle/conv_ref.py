"""Float64 CPU oracle for the causal temporal convolution with a carried
last-frame cache.

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the CPU-baseline leg of the benchmark may import or run it. It
shares no code with the CUDA path.

Where it comes from
-------------------
The SANA-Video ICLR 2026 oral transcript (shadowingenglish.com), the part on
the causal FFN with temporal convolution (after the block KV cache part):

  * the model adds a temporal convolution to its feed-forward block for
    temporal modelling;
  * under block-causal training a block must not see the next block, so a
    zero token is padded between two blocks;
  * a block must still see the previous block, so the last token of block i
    is cached and used as the first token seen by block i+1;
  * the zero padding token is removed afterwards, so it never reaches the
    output.

The talk gives no kernel size or layout. The reading taken here is the
plainest one that needs exactly one cached frame and exactly one padding
frame: a depthwise convolution along the frame axis with three taps, centred
on the current frame (one frame of context on each side). Per channel c,
frame t and spatial token s:

    y[t] = w[c,0] * x_prev + w[c,1] * x[t] + w[c,2] * x_next + bias[c]

    x_prev = x[t-1]        (for the first frame of a block this is the last
                            frame of the previous block: the cached token;
                            for the first frame of the call it is the cache
                            handed in, zero at the start of a video)
    x_next = x[t+1]        inside a block, and 0 for the last frame of a
                            block (the padding token between blocks)

Blocks hold `frames_per_block` frames, counted from the first frame of the
call; a shorter last block ends the call. The cache handed on is the last
frame of the call. Everything runs in float64.
"""
from __future__ import annotations

import numpy as np

__all__ = ["temporal_conv_ref"]


def temporal_conv_ref(x, w, bias=None, cache=None, frames_per_block=None):
    """Causal temporal convolution over the frames of x.

    x : [..., T, S, C]   any float dtype, widened to float64
    w : [C, 3]           taps for the previous, current and next frame
    bias : [C] or None
    cache : [..., S, C] or None   the frame before x[..., 0, :, :] (None: zeros)
    frames_per_block : frames per block (None: one block of all T frames)

    Returns (y [..., T, S, C] float64, cache_out = x[..., T-1, :, :] float64).
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    *lead, T, S, C = x.shape
    F = T if frames_per_block is None else int(frames_per_block)
    if F < 1:
        raise ValueError("frames_per_block must be >= 1")
    if w.shape != (C, 3):
        raise ValueError("w must be [C, 3]")
    b = np.zeros(C) if bias is None else np.asarray(bias, dtype=np.float64)
    prev0 = np.zeros(tuple(lead) + (S, C)) if cache is None else np.asarray(cache, np.float64)
    y = np.empty_like(x)
    for t in range(T):
        last_in_block = (t + 1) % F == 0 or t == T - 1
        x_prev = prev0 if t == 0 else x[..., t - 1, :, :]
        x_next = np.zeros_like(x[..., t, :, :]) if last_in_block else x[..., t + 1, :, :]
        y[..., t, :, :] = w[:, 0] * x_prev + w[:, 1] * x[..., t, :, :] + w[:, 2] * x_next + b
    return y, x[..., T - 1, :, :].copy()
