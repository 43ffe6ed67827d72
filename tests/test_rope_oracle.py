"""The 3D RoPE oracle against its pins (tests/rope_pins.py), and plausible
mistakes planted in a copy of it, on the CPU, each caught by a pin."""
import numpy as np
import pytest

import rope_pins
from oracle import rope3d_ref


@pytest.mark.parametrize("name", sorted(rope_pins.ALL))
def test_rope_pin(name):
    rope_pins.ALL[name](rope3d_ref)


def _variant(sections=None, pos=None, pairs="adjacent", sign=1.0, base=10000.0, t_from_call=False):
    """A copy of the oracle's steps with one rule changed."""
    def rope(x, grid_w, t0=0):
        x = np.asarray(x, np.float64)
        T, S, D = x.shape[-3:]
        dh = 2 * (D // 6)
        secs = sections(D) if sections else (D - 2 * dh, dh, dh)
        r = np.arange(S)
        t = np.arange(T)[:, None] + (0 if t_from_call else t0) + np.zeros((1, S))
        h = np.broadcast_to(r // grid_w, (T, S))
        w = np.broadcast_to(r % grid_w, (T, S))
        if pos:
            t, h, w = pos(t, h, w)
        angs = []
        for p, size in zip((t, h, w), secs):
            i = np.arange(size // 2)
            angs.append(p[..., None] * base ** (-2.0 * i / size))
        a = np.concatenate(angs, axis=-1)
        c, s = np.cos(a), sign * np.sin(a)
        out = np.empty_like(x)
        if pairs == "adjacent":
            xe, xo = x[..., 0::2], x[..., 1::2]
            out[..., 0::2] = xe * c - xo * s
            out[..., 1::2] = xe * s + xo * c
        else:                                   # rotate-half pairing (i, i + D/2)
            xe, xo = x[..., : D // 2], x[..., D // 2:]
            out[..., : D // 2] = xe * c - xo * s
            out[..., D // 2:] = xe * s + xo * c
        return out
    return rope


MUTANTS = {
    "equal_thirds_rounded": _variant(sections=lambda D: (2 * (D // 6), D - 4 * (D // 6), 2 * (D // 6))),
    "h_w_swapped": _variant(pos=lambda t, h, w: (t, w, h)),
    "rotate_half_pairs": _variant(pairs="half"),
    "clockwise": _variant(sign=-1.0),
    "base_1000": _variant(base=1000.0),
    "frame_index_relative_to_call": _variant(t_from_call=True),
}


def test_unmutated_copy_passes_every_pin():
    ok = _variant()
    for check in rope_pins.ALL.values():
        check(ok)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_each_planted_mistake_fails_a_pin(mutant):
    rope = MUTANTS[mutant]
    failed = []
    for name, check in rope_pins.ALL.items():
        try:
            check(rope)
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught the planted mistake {mutant!r}"
