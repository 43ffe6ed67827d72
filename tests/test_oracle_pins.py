"""The float64 oracle against facts it does not define itself (see tests/pins.py)."""
import json
import math
import os

import numpy as np
import pytest

import pins
from oracle import gdn_scan_ref, rel_frobenius, default_key_scale

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("name", sorted(pins.ALL))
def test_pin(name):
    pins.ALL[name](gdn_scan_ref)


def test_stability_961_frames():
    pins.check_stability(gdn_scan_ref)


def test_default_key_scale():
    assert default_key_scale(64, 880) == 1.0 / math.sqrt(64 * 880)


def test_scalar_worked_example():
    """Hand-derived scalar case (D = S = 1, so s = 1): see the fixture's notes."""
    with open(os.path.join(GOLDEN, "scalar_worked_example.json")) as f:
        ex = json.load(f)
    T = len(ex["gamma"])
    q = np.array(ex["q"], float).reshape(T, 1, 1)
    k = np.array(ex["k"], float).reshape(T, 1, 1)
    v = np.array(ex["v"], float).reshape(T, 1, 1)
    o, m = gdn_scan_ref(q, k, v, ex["gamma"], ex["beta"], state_in=np.array([[ex["m0"]]]))
    assert np.allclose(o.reshape(T), ex["out"], rtol=0, atol=1e-15)
    assert abs(m[0, 0] - ex["state"][-1]) < 1e-15


def test_tiny_fixture_regression():
    """The committed fixture was written by tests/golden/make_golden.py from the oracle."""
    path = os.path.join(GOLDEN, "tiny_d4_s6_t3.json")
    with open(path) as f:
        fx = json.load(f)
    inp = {k: np.array(v) for k, v in fx["inputs"].items()}
    o, m = gdn_scan_ref(inp["q"], inp["k"], inp["v"], inp["gamma"], inp["beta"],
                        state_in=inp["state_in"])
    assert np.max(np.abs(o - np.array(fx["out"]))) < 1e-13
    assert np.max(np.abs(m - np.array(fx["state_out"]))) < 1e-13


def test_rel_frobenius_floor():
    ref = np.zeros((2, 3, 3))
    ref[1] = 1.0
    x = ref.copy()
    x[0, 0, 0] = 1e-6
    e = rel_frobenius(x, ref)
    assert e[1] == 0.0 and abs(e[0] - 1e-6 / 3.0) < 1e-18


def test_batched_equals_per_head():
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((2, 3, 4, 5, 6)) for _ in range(3))
    g = rng.uniform(0.5, 1, (2, 3, 4))
    b = rng.uniform(0, 1, (2, 3, 4))
    o, m = gdn_scan_ref(q, k, v, g, b)
    for i in range(2):
        for j in range(3):
            o1, m1 = gdn_scan_ref(q[i, j], k[i, j], v[i, j], g[i, j], b[i, j])
            assert np.array_equal(o1, o[i, j]) and np.array_equal(m1, m[i, j])
