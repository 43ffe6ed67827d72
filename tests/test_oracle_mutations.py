"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each one."""
import math

import pytest

import pins
import oracle.gdn_ref as ref


def _mut_no_gamma_in_residual(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - K @ M if delta else v
    M2 = g * M + b * (K.T @ R)
    return M2, q @ M2


def _mut_preupdate_readout(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = g * M + b * (K.T @ R)
    return M2, q @ M


def _mut_no_decay(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = M + b * (K.T @ R)
    return M2, q @ M2


def _mut_scale_once(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = g * M + b * (k.T @ R)
    return M2, q @ M2


def _mut_transposed_prediction(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M.T) if delta else v
    M2 = g * M + b * (K.T @ R)
    return M2, q @ M2


def _mut_swapped_gates(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - b * (K @ M) if delta else v
    M2 = b * M + g * (K.T @ R)
    return M2, q @ M2


def _mut_no_beta(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = g * M + (K.T @ R)
    return M2, q @ M2


def _mut_residual_sign(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v + g * (K @ M) if delta else v
    M2 = g * M + b * (K.T @ R)
    return M2, q @ M2


def _mut_transposed_readout(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = g * M + b * (K.T @ R)
    return M2, q @ M2.T


def _mut_decay_inside_update(M, q, k, v, g, b, s, delta):
    K = s * k
    R = v - g * (K @ M) if delta else v
    M2 = g * (M + b * (K.T @ R))
    return M2, q @ M2


MUTANTS = {f.__name__[5:]: f for f in [
    _mut_no_gamma_in_residual, _mut_preupdate_readout, _mut_no_decay, _mut_scale_once,
    _mut_transposed_prediction, _mut_swapped_gates, _mut_no_beta, _mut_residual_sign,
    _mut_transposed_readout, _mut_decay_inside_update]}


def _caught(scan):
    failures = []
    for name, check in pins.ALL.items():
        try:
            check(scan)
        except AssertionError:
            failures.append(name)
    return failures


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    monkeypatch.setattr(ref, "_frame_step", MUTANTS[name])
    assert _caught(ref.gdn_scan_ref), f"mutant {name} passed every pin"


@pytest.mark.parametrize("wrong", ["sqrt_d", "sqrt_s"])
def test_wrong_default_scale_is_caught(wrong, monkeypatch):
    f = {"sqrt_d": lambda D, S: 1.0 / math.sqrt(D), "sqrt_s": lambda D, S: 1.0 / math.sqrt(S)}[wrong]
    monkeypatch.setattr(ref, "default_key_scale", f)
    assert _caught(ref.gdn_scan_ref)


def test_unmutated_passes_all():
    assert _caught(ref.gdn_scan_ref) == []
