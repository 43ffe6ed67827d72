"""Float64 CPU oracle for the frame-wise Gated DeltaNet (GDN) scan.

TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline leg
of the benchmark may import or run this module; the library never does. It
shares no code with the CUDA path.

What it computes, and where that comes from
-------------------------------------------
"NVIDIA Apresenta SANA-WM: Um Modelo de Mundo de Larga Escala ..."
(acheiumaia.com.br), section "A Arquitetura: Quatro Decisões de Design
Centrais", item "1. Atenção Linear Híbrida com Gated DeltaNet (GDN)":

  * one whole latent frame (S spatial tokens) is one recurrent step;
  * the recurrent state has the constant size D x D, whatever the video length;
  * a decay gate gamma lowers the weight of stale past frames;
  * a delta-rule correction writes only the residual between the target value
    and what the current state predicts;
  * keys are scaled by 1/sqrt(D*S) (D = head dim, S = spatial tokens per frame)
    so the transition matrix keeps a bounded spectral norm.

The article gives these facts in prose only. The update is fixed, exactly and
for both this oracle and the GPU path, as the plainest reading of them. Per
head and frame t, with K_t, Q_t, V_t in R^{S x D}, s = 1/sqrt(D*S), M in
R^{D x D} (rows: key dimension, columns: value dimension):

    K  = s * K_t
    W  = K @ M_{t-1}                  prediction of the values by the current state
    R  = V_t - gamma_t * W            residual w.r.t. the decayed state's prediction
    M_t = gamma_t * M_{t-1} + beta_t * K^T @ R
    O_t = Q_t @ M_t                   read-out with the updated state

The "cumulative" mode (delta=False) replaces R by V_t. With gamma = beta = 1
it is the block-causal linear attention of the SANA-Video talk
("SANA-Video ... ICLR 2026 oral", shadowingenglish.com transcript, the part on
block causal linear attention): the state of block i is the state of block
i-1 plus block i's K^T V, with a fixed D x D shape.

Precision: every input is widened exactly to float64 and every step runs in
float64. The step order above is the order of the definition; numpy matmul is
the only library primitive used.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["default_key_scale", "gdn_scan_ref", "rel_frobenius"]


def default_key_scale(D: int, S: int) -> float:
    """s = 1/sqrt(D*S), the key scale of the SANA-WM article (GDN item)."""
    return 1.0 / math.sqrt(float(D) * float(S))


def _frame_step(M, q, k, v, gamma, beta, s, delta):
    """One frame of one head, in the definition's order. Returns (M_t, O_t)."""
    K = s * k
    if delta:
        W = K @ M
        R = v - gamma * W
    else:
        R = v
    M_new = gamma * M + beta * (K.T @ R)
    O = q @ M_new
    return M_new, O


def gdn_scan_ref(q, k, v, gamma, beta, state_in=None, key_scale=None, delta=True,
                 return_states=False):
    """Run the frame-wise GDN recurrence over T frames.

    q, k, v : [..., T, S, D]   any float dtype, widened to float64
    gamma, beta : [..., T]
    state_in : [..., D, D] or None (None means M_0 = 0)
    key_scale : None for 1/sqrt(D*S), else the scale to use (tests only)
    delta : False gives the cumulative (no delta correction) form
    return_states : also return every M_t as [..., T, D, D]

    Returns (O [..., T, S, D] float64, M_T [..., D, D] float64[, states]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    *lead, T, S, D = q.shape
    s = default_key_scale(D, S) if key_scale is None else float(key_scale)
    lead = tuple(lead)
    n = int(np.prod(lead)) if lead else 1
    qf = q.reshape(n, T, S, D)
    kf = k.reshape(n, T, S, D)
    vf = v.reshape(n, T, S, D)
    gf = gamma.reshape(n, T)
    bf = beta.reshape(n, T)
    if state_in is None:
        m0 = np.zeros((n, D, D))
    else:
        m0 = np.asarray(state_in, dtype=np.float64).reshape(n, D, D)
    out = np.empty((n, T, S, D))
    m_last = np.empty((n, D, D))
    states = np.empty((n, T, D, D)) if return_states else None
    for i in range(n):
        M = m0[i].copy()
        for t in range(T):
            M, out[i, t] = _frame_step(M, qf[i, t], kf[i, t], vf[i, t], gf[i, t], bf[i, t],
                                       s, delta)
            if return_states:
                states[i, t] = M
        m_last[i] = M
    res = (out.reshape(lead + (T, S, D)), m_last.reshape(lead + (D, D)))
    if return_states:
        res = res + (states.reshape(lead + (T, D, D)),)
    return res


def rel_frobenius(x, ref, axes=(-2, -1), floor=1e-30):
    """Relative Frobenius error per leading index: ||x - ref||_F / ||ref||_F over `axes`.

    Where ||ref||_F < floor, the absolute error divided by the largest reference
    norm along the same array is returned instead.
    """
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.sqrt(np.sum((x - ref) ** 2, axis=axes))
    den = np.sqrt(np.sum(ref ** 2, axis=axes))
    big = max(float(np.max(den)) if den.size else 0.0, floor)
    return np.where(den >= floor, num / np.maximum(den, floor), num / big)
