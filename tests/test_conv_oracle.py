"""The temporal-convolution oracle against its pins (tests/conv_pins.py), and
plausible mistakes planted in a copy of it, on the CPU, each caught by a pin."""
import numpy as np
import pytest

import conv_pins
from oracle import temporal_conv_ref


@pytest.mark.parametrize("name", sorted(conv_pins.ALL))
def test_conv_pin(name):
    conv_pins.ALL[name](temporal_conv_ref)


def _make(prev_rule, next_rule, taps=(0, 1, 2), bias=True, cache_out_last=True):
    """A variant of the oracle's loop with one rule changed."""
    def conv(x, w, b=None, cache=None, frames_per_block=None):
        x = np.asarray(x, np.float64)
        w = np.asarray(w, np.float64)
        T, S, C = x.shape
        F = T if frames_per_block is None else int(frames_per_block)
        bb = np.zeros(C) if (b is None or not bias) else np.asarray(b, np.float64)
        c0 = np.zeros((S, C)) if cache is None else np.asarray(cache, np.float64)
        y = np.empty_like(x)
        for t in range(T):
            xp = prev_rule(x, t, F, c0)
            xn = next_rule(x, t, F, T)
            y[t] = w[:, taps[0]] * xp + w[:, taps[1]] * x[t] + w[:, taps[2]] * xn + bb
        return y, (x[T - 1] if cache_out_last else x[0]).copy()
    return conv


def _prev_ok(x, t, F, c0):
    return c0 if t == 0 else x[t - 1]


def _next_ok(x, t, F, T):
    return np.zeros_like(x[t]) if ((t + 1) % F == 0 or t == T - 1) else x[t + 1]


MUTANTS = {
    # the next block leaks in: no zero token between blocks
    "no_pad": _make(_prev_ok, lambda x, t, F, T: np.zeros_like(x[t]) if t == T - 1 else x[t + 1]),
    # every block starts from zero instead of the previous block's last frame
    "no_cached_token": _make(lambda x, t, F, c0: (c0 if t == 0 else np.zeros_like(x[t]))
                             if t % F == 0 else x[t - 1], _next_ok),
    # the cache handed in is ignored
    "cache_ignored": _make(lambda x, t, F, c0: np.zeros_like(x[0]) if t == 0 else x[t - 1], _next_ok),
    # previous and next taps swapped
    "taps_reversed": _make(_prev_ok, _next_ok, taps=(2, 1, 0)),
    # bias dropped
    "no_bias": _make(_prev_ok, _next_ok, bias=False),
    # the pad placed after a block's first frame instead of its last
    "pad_off_by_one": _make(_prev_ok, lambda x, t, F, T: np.zeros_like(x[t])
                            if (t % F == 0 or t == T - 1) else x[t + 1]),
    # the cache handed on is the call's first frame
    "wrong_cache_out": _make(_prev_ok, _next_ok, cache_out_last=False),
}


def test_unmutated_copy_passes_every_pin():
    ok = _make(_prev_ok, _next_ok)
    for name, check in conv_pins.ALL.items():
        check(ok)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(mutant):
    conv = MUTANTS[mutant]
    failed = []
    for name, check in conv_pins.ALL.items():
        try:
            check(conv)
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught the planted mistake {mutant!r}"
