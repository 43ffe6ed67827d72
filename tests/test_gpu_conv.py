"""The causal temporal convolution (gdn_temporal_conv) against the float64
oracle, through the C ABI.

Bound, element by element: the kernel evaluates three products and the bias
in fp32 (at most four roundings, each within 2^-24 of the running sum, so
within 2^-22 of the sum of the terms' magnitudes) and rounds y to bf16 (8
significant bits: within 2^-8 of the value), so
    |y - y_ref| <= 2^-8 |y_ref| + 2^-21 (|w0 x_prev| + |w1 x| + |w2 x_next| + |bias|).
"""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from oracle import rel_frobenius, temporal_conv_ref

pytestmark = pytest.mark.gpu


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def _magnitude(x, w, bias, cache, F):
    """Sum of the terms' magnitudes, per output element (the oracle with |.|)."""
    return temporal_conv_ref(np.abs(x), np.abs(w), np.abs(bias), None if cache is None else
                             np.abs(cache), F)[0]


def _check(y, x, w, bias, cache, F):
    ref, ref_cache = temporal_conv_ref(x, w, bias, cache, F)
    got = y.float().cpu().numpy().astype(np.float64)
    mag = _magnitude(x, w, bias, cache, F)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -21 * mag
    excess = np.abs(got - ref) - bound
    assert np.all(np.isfinite(got))
    assert float(np.max(excess)) <= 0.0, f"bound exceeded by {float(np.max(excess)):.3e}"
    e = float(np.max(rel_frobenius(got.reshape(-1, *got.shape[-2:]), ref.reshape(-1, *ref.shape[-2:]))))
    assert e <= 2e-2
    return ref_cache


@pytest.mark.parametrize("B,T,S,C,F", [
    (1, 1, 1, 8, 1), (1, 2, 3, 8, 1), (2, 5, 7, 24, 2), (1, 17, 33, 64, 3),
    (2, 40, 5, 256, 8), (1, 9, 2, 16, 100), (1, 300, 4, 64, 7), (3, 64, 1, 8, 5),
])
@pytest.mark.parametrize("with_cache", [False, True])
def test_conv_against_oracle(B, T, S, C, F, with_cache):
    wl = inputs.ConvWorkload("c", B, T, S, C, F, 700 + T + S + C)
    x = inputs.conv_full(wl)
    w, bias = inputs.conv_params(wl)
    cache = inputs.conv_cache(wl) if with_cache else None
    y, c_out = gdn.temporal_conv(_dev_bf16(x), torch.from_numpy(w).cuda(),
                                 torch.from_numpy(bias).cuda(),
                                 None if cache is None else _dev_bf16(cache), frames_per_block=F)
    torch.cuda.synchronize()
    ref_cache = _check(y, x, w, bias, cache, F)
    assert np.array_equal(c_out.float().cpu().numpy(), ref_cache)


def test_conv_without_bias():
    wl = inputs.ConvWorkload("nb", 1, 6, 3, 16, 4, 750)
    x = inputs.conv_full(wl)
    w, _ = inputs.conv_params(wl)
    y, _ = gdn.temporal_conv(_dev_bf16(x), torch.from_numpy(w).cuda(), None, None, frames_per_block=4)
    torch.cuda.synchronize()
    _check(y, x, w, np.zeros(16, np.float32), None, 4)


def test_conv_split_calls_equal_one_call_and_in_place_cache():
    """Calls over whole blocks that carry the cache (in place) give exactly one call's y."""
    wl = inputs.ConvWorkload("split", 2, 24, 9, 40, 4, 751)
    x = _dev_bf16(inputs.conv_full(wl))
    w, bias = (torch.from_numpy(a).cuda() for a in inputs.conv_params(wl))
    c0 = _dev_bf16(inputs.conv_cache(wl))
    y_all, c_all = gdn.temporal_conv(x, w, bias, c0, frames_per_block=4)
    cache = c0.clone()
    parts = []
    for a, b in ((0, 8), (8, 12), (12, 24)):
        y, _ = gdn.temporal_conv(x[:, a:b].contiguous(), w, bias, cache, frames_per_block=4,
                                 cache_out=cache)
        parts.append(y)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), y_all)
    assert torch.equal(cache, c_all)


def test_conv_bad_arguments():
    x = torch.zeros((1, 2, 3, 12), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((12, 3), device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.temporal_conv(x, w)
    assert ei.value.status == -2        # C not a multiple of 8
    x = torch.zeros((1, 2, 3, 16), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 3), device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.temporal_conv(x, w, frames_per_block=0)
    assert ei.value.status == -2
    with pytest.raises(gdn.GdnError) as ei:
        gdn.temporal_conv(x, w, y=x)
    assert ei.value.status == -7        # y overlaps x


@pytest.mark.slow
def test_conv_full_size_sampled_columns():
    """The rollout-shaped workload (961 frames, 880 tokens, 2048 channels) in the
    launch bench.py times; sampled tokens checked over every frame."""
    wl = inputs.CONV_WORKLOADS["conv_rollout"]
    x = torch.empty((wl.B, wl.T, wl.S, wl.C), dtype=torch.bfloat16, device="cuda")
    tokens = [0, 437, 879]
    host = np.empty((wl.T, len(tokens), wl.C), np.float32)
    for t in range(wl.T):
        f = inputs.conv_frame(wl, 0, t)
        x[0, t].copy_(torch.from_numpy(f).to(torch.bfloat16))
        host[t] = f[tokens]
    w, bias = inputs.conv_params(wl)
    c0 = inputs.conv_cache(wl)
    y, c_out = gdn.temporal_conv(x, torch.from_numpy(w).cuda(), torch.from_numpy(bias).cuda(),
                                 _dev_bf16(c0), frames_per_block=wl.F)
    torch.cuda.synchronize()
    ys = y[0][:, tokens].contiguous()[None]
    _check(ys, host[None], w, bias, c0[:, tokens], wl.F)
    assert torch.equal(c_out[0], x[0, -1])
