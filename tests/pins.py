"""Checks that pin the float64 oracle to facts other than itself.

Each check takes `scan`, a function with the signature of
oracle.gdn_ref.gdn_scan_ref, and raises AssertionError on failure. The facts:

  cumulative   gamma=1, beta=1 without the delta correction is block-causal
               linear attention (SANA-Video talk, block causal linear
               attention: the state is the running sum of the blocks' K^T V);
               checked against the attention written in score form, with no
               state at all.
  decayed      the same with per-frame gamma and beta: each past frame tau is
               weighted by beta_tau times the gammas of the later frames.
  literal      gamma=1, beta=0 leaves any state untouched.
  t1           one frame equals the closed form
               M_1 = gamma (I - beta s^2 K^T K) M_0 + beta s K^T V, and with
               M_0 = 0 the read-out is beta s (Q K^T) V, evaluated score-first.
  decay        beta=0 scales the state by the product of the gammas.
  fixed_point  gamma=1 and V_t equal to the state's own prediction leaves the
               state unchanged (the delta rule writes only the residual).
  transition   over many frames the state follows M_t = A_t M_{t-1} + c_t with
               A_t = gamma_t (I - beta_t s^2 K_t^T K_t), c_t = beta_t s K_t^T V_t.
  stability    with keys of unit rows and the 1/sqrt(D S) scale the state
               stays finite and under the bound the contraction gives, over
               961 frames; without the scale it blows up (SANA-WM article, GDN
               item: the key scale bounds the transition's spectral norm).
  split        a scan split into two calls that carry the state equals one call.
  scale        the default key scale is 1/sqrt(D S), not 1/sqrt(D) or 1/sqrt(S).
"""
from __future__ import annotations

import math

import numpy as np


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _rel(x, y):
    d = float(np.linalg.norm(np.asarray(x) - np.asarray(y)))
    n = float(np.linalg.norm(np.asarray(y)))
    return d / max(n, 1e-300)


def check_cumulative(scan, seed=11, T=5, S=7, D=4):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    o, _ = scan(q, k, v, np.ones(T), np.ones(T), delta=False)
    s = 1.0 / math.sqrt(D * S)
    for t in range(T):
        kk = s * k[: t + 1].reshape(-1, D)          # all keys seen so far, scaled
        vv = v[: t + 1].reshape(-1, D)
        ref = (q[t] @ kk.T) @ vv                     # scores first, no state
        assert _rel(o[t], ref) < 1e-12, ("cumulative", t, _rel(o[t], ref))


def check_decayed(scan, seed=12, T=6, S=5, D=3):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    g = rng.uniform(0.5, 1.0, T)
    b = rng.uniform(0.1, 1.0, T)
    o, _ = scan(q, k, v, g, b, delta=False)
    s = 1.0 / math.sqrt(D * S)
    for t in range(T):
        ref = np.zeros((S, D))
        for tau in range(t + 1):
            w = b[tau] * np.prod(g[tau + 1: t + 1])
            ref += w * ((q[t] @ (s * k[tau]).T) @ v[tau])
        assert _rel(o[t], ref) < 1e-12, ("decayed", t, _rel(o[t], ref))


def check_literal(scan, seed=13, T=4, S=6, D=5):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    m0 = _rand(rng, D, D)
    o, mt = scan(q, k, v, np.ones(T), np.zeros(T), state_in=m0)
    assert np.array_equal(mt, m0), "literal: state changed"
    for t in range(T):
        assert _rel(o[t], q[t] @ m0) < 1e-15, ("literal", t)


def check_t1(scan, seed=14, S=9, D=4):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, 1, S, D), _rand(rng, 1, S, D), _rand(rng, 1, S, D)
    m0 = _rand(rng, D, D)
    g, b = np.array([0.8]), np.array([0.6])
    s = 1.0 / math.sqrt(D * S)
    o, m1 = scan(q, k, v, g, b, state_in=m0)
    K, V = k[0], v[0]
    ref = g[0] * (np.eye(D) - b[0] * s * s * (K.T @ K)) @ m0 + b[0] * s * (K.T @ V)
    assert _rel(m1, ref) < 1e-12, ("t1 state", _rel(m1, ref))
    assert _rel(o[0], q[0] @ ref) < 1e-12, "t1 out"
    o0, _ = scan(q, k, v, g, b)
    ref0 = b[0] * s * ((q[0] @ K.T) @ V)
    assert _rel(o0[0], ref0) < 1e-12, ("t1 zero-state out", _rel(o0[0], ref0))


def check_decay(scan, seed=15, T=7, S=4, D=3):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    m0 = _rand(rng, D, D)
    g = rng.uniform(0.3, 1.0, T)
    o, mt, states = scan(q, k, v, g, np.zeros(T), state_in=m0, return_states=True)
    for t in range(T):
        p = np.prod(g[: t + 1])
        assert _rel(states[t], p * m0) < 1e-13, ("decay state", t)
        assert _rel(o[t], p * (q[t] @ m0)) < 1e-13, ("decay out", t)


def check_fixed_point(scan, seed=16, T=5, S=8, D=4):
    rng = np.random.default_rng(seed)
    s = 1.0 / math.sqrt(D * S)
    M = _rand(rng, D, D)
    for t in range(T):
        q = _rand(rng, 1, S, D)
        k = _rand(rng, 1, S, D)
        v = (s * k[0] @ M)[None]                     # exactly what the state predicts
        b = np.array([rng.uniform(0.1, 1.0)])
        _, M2 = scan(q, k, v, np.ones(1), b, state_in=M)
        assert _rel(M2, M) < 1e-13, ("fixed point", t, _rel(M2, M))
        M = M2


def check_transition(scan, seed=17, T=10, S=12, D=5):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    g = rng.uniform(0.5, 1.0, T)
    b = rng.uniform(0.0, 1.0, T)
    m0 = _rand(rng, D, D)
    s = 1.0 / math.sqrt(D * S)
    o, mt, states = scan(q, k, v, g, b, state_in=m0, return_states=True)
    M = m0
    for t in range(T):
        A = g[t] * (np.eye(D) - b[t] * s * s * (k[t].T @ k[t]))
        c = b[t] * s * (k[t].T @ v[t])
        M = A @ M + c
        assert _rel(states[t], M) < 1e-12, ("transition state", t, _rel(states[t], M))
        assert _rel(o[t], q[t] @ M) < 1e-12, ("transition out", t)
    assert _rel(mt, M) < 1e-12


def check_stability(scan, seed=18, T=961, S=880, D=64):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, S, D))
    k = rng.standard_normal((T, S, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, S, D))
    g = rng.uniform(0.95, 1.0, T)
    b = rng.uniform(0.2, 1.0, T)
    s = 1.0 / math.sqrt(D * S)
    _, _, states = scan(q, k, v, g, b, return_states=True)
    assert np.all(np.isfinite(states)), "scaled keys gave a non-finite state"
    # ||A_t||_2 <= gamma_t when beta_t s^2 ||K^T K|| <= 2 (here <= 1/D), so
    # ||M_t|| <= gamma_t ||M_{t-1}|| + ||c_t||.
    bound = 0.0
    for t in range(T):
        assert b[t] * s * s * np.linalg.norm(k[t].T @ k[t], 2) <= 1.0 / D + 1e-12
        bound = g[t] * bound + b[t] * s * np.linalg.norm(k[t].T @ v[t], 2)
        assert np.linalg.norm(states[t], 2) <= bound * (1 + 1e-9), ("bound", t)
    with np.errstate(over="ignore", invalid="ignore"):
        _, _, raw = scan(q, k, v, g, b, key_scale=1.0, return_states=True)
    mags = np.abs(raw).reshape(T, -1).max(axis=1)
    blown = ~np.isfinite(mags) | (mags > 1e300)
    assert blown.any(), "unscaled keys did not blow up within 961 frames"


def check_split(scan, seed=19, T=9, S=6, D=4):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, T, S, D), _rand(rng, T, S, D), _rand(rng, T, S, D)
    g = rng.uniform(0.5, 1.0, T)
    b = rng.uniform(0.0, 1.0, T)
    o, mt = scan(q, k, v, g, b)
    for cut in (1, 4, T - 1):
        o1, m1 = scan(q[:cut], k[:cut], v[:cut], g[:cut], b[:cut])
        o2, m2 = scan(q[cut:], k[cut:], v[cut:], g[cut:], b[cut:], state_in=m1)
        assert np.array_equal(np.concatenate([o1, o2]), o), ("split out", cut)
        assert np.array_equal(m2, mt), ("split state", cut)


def check_scale(scan, seed=20, S=6, D=4):
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, 1, S, D), _rand(rng, 1, S, D), _rand(rng, 1, S, D)
    g, b = np.array([0.9]), np.array([0.7])
    o_default, m_default = scan(q, k, v, g, b)
    o_exp, m_exp = scan(q, k, v, g, b, key_scale=1.0 / math.sqrt(D * S))
    assert _rel(m_default, m_exp) < 1e-15
    for wrong in (1.0 / math.sqrt(D), 1.0 / math.sqrt(S), 1.0 / (D * S)):
        _, m_w = scan(q, k, v, g, b, key_scale=wrong)
        assert _rel(m_w, m_default) > 1e-3


ALL = {
    "cumulative": check_cumulative,
    "decayed": check_decayed,
    "literal": check_literal,
    "t1": check_t1,
    "decay": check_decay,
    "fixed_point": check_fixed_point,
    "transition": check_transition,
    "split": check_split,
    "scale": check_scale,
}
