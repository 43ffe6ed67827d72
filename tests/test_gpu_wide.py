"""The all-SM scan (gdn_wide.cu) through the C ABI.

It runs the arithmetic of the cluster kernel (same operands, same MMAs in the
same order, same fp32 epilogue), only on other SMs, so its outputs and final
states must equal the cluster kernel's bit for bit; both are also compared
with the float64 oracle within 2e-2 per frame and head.
"""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, oracle_head, to_np64

pytestmark = pytest.mark.gpu


def _scan(monkeypatch, wide, P, q, k, v, g, be, st=None, state_out=None, delta=True):
    monkeypatch.setenv("GDN_WIDE", "1" if wide else "0")
    if P:
        monkeypatch.setenv("GDN_WIDE_P", str(P))
    else:
        monkeypatch.delenv("GDN_WIDE_P", raising=False)
    B, H, T, S, D = q.shape
    kern, ctas = gdn.plan(B, H, T, S, D)
    if wide:
        assert kern == gdn.KERNEL_TC_WIDE and (not P or ctas == P)
    else:
        assert kern == gdn.KERNEL_TC
    out, s = gdn.frame_scan(q, k, v, g, be, st, state_out=state_out, delta=delta)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return out, s


def _check(monkeypatch, wl, P, heads=None, state=False, delta=True):
    q, k, v, g, be = device_workload(wl)
    st = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda() if state else None
    o_w, s_w = _scan(monkeypatch, True, P, q, k, v, g, be, st, delta=delta)
    o_c, s_c = _scan(monkeypatch, False, 0, q, k, v, g, be, st, delta=delta)
    assert torch.equal(o_w, o_c), "outputs differ from the cluster kernel"
    assert torch.equal(s_w, s_c), "final states differ from the cluster kernel"
    heads = heads or [(b, h) for b in range(wl.B) for h in range(wl.H)]
    for b, h in heads:
        ro, rs = oracle_head(wl, b, h, None, None if st is None else st[b, h].cpu().numpy(), delta)
        assert_close(to_np64(o_w[b, h]), ro, to_np64(s_w[b, h]), rs, TOL_BF16, f"{wl.name} b{b} h{h}")


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("S", [1, 65, 200])
def test_wide_shapes_and_head_ctas(monkeypatch, S, P):
    wl = inputs.Workload(f"wide_s{S}", 1, 3, 64, 5, S, "bf16", 700 + S, "gauss", "tiny")
    _check(monkeypatch, wl, P)


@pytest.mark.parametrize("T", [2, 17, 40])
def test_wide_ring_reuse(monkeypatch, T):
    """More frames than ring slots: producers wait for the slot's previous frame."""
    wl = inputs.Workload(f"wide_t{T}", 2, 3, 64, T, 300, "bf16", 710 + T, "l2", "rollout")
    _check(monkeypatch, wl, 0, state=True)


def test_wide_no_delta(monkeypatch):
    wl = inputs.Workload("wide_nodelta", 1, 4, 64, 20, 130, "bf16", 720, "l2", "rollout")
    _check(monkeypatch, wl, 2, delta=False)


def test_wide_in_place_state(monkeypatch):
    """state_in is state_out: rank 0 writes the final state only after every CTA
    of its head has read the initial one."""
    wl = inputs.Workload("wide_inplace", 1, 5, 64, 3, 250, "bf16", 730, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    ref_o, ref_s = _scan(monkeypatch, False, 0, q, k, v, g, be, m0.clone())
    st = m0.clone()
    o, s = _scan(monkeypatch, True, 8, q, k, v, g, be, st, state_out=st)
    assert s.data_ptr() == st.data_ptr()
    assert torch.equal(o, ref_o) and torch.equal(st, ref_s)


def test_wide_many_heads(monkeypatch):
    """More heads than fit 2 CTAs each: one head CTA per head, few helpers."""
    wl = inputs.Workload("wide_heads", 4, 25, 64, 4, 96, "bf16", 740, "gauss", "short")
    _check(monkeypatch, wl, 0, heads=[(0, 0), (3, 24), (2, 11)])


def test_wide_rollout_sampled_heads(monkeypatch):
    """The 961-frame rollout (B=1, H=32, S=880): equal to the cluster kernel,
    and sampled heads against the oracle."""
    wl = inputs.WORKLOADS["rollout"]
    q, k, v, g, be = inputs.device_draw(wl, torch.device("cuda", 0))
    o_w, s_w = _scan(monkeypatch, True, 0, q, k, v, g, be)
    o_c, s_c = _scan(monkeypatch, False, 0, q, k, v, g, be)
    assert torch.equal(o_w, o_c) and torch.equal(s_w, s_c)
    del o_c, s_c
