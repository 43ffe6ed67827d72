"""The row-split single-frame kernel (gdn_frame_step, D = 64, bf16) against the
float64 oracle, through the C ABI.

A cluster of 2 or 4 CTAs shares each head's frame by rows, so the cases cover
frames that leave some CTAs without rows (S < 32 * P), ragged last boxes,
frames at the kernel's row limit, and more heads than fit on the GPU at once.
Tolerance: relative Frobenius error 2e-2 per head for out and the new state.
"""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, to_np64
from oracle import gdn_scan_ref

pytestmark = pytest.mark.gpu


def _frame0(x):
    return x[:, :, 0].contiguous()


def _step_and_compare(wl, state_scale=0.5, delta=True, gates=None):
    q, k, v, g, be = device_workload(wl)
    if gates is not None:
        g = torch.full_like(g, gates[0])
        be = torch.full_like(be, gates[1])
    m0 = inputs.state(wl, scale=state_scale)
    out, st = gdn.frame_step(_frame0(q), _frame0(k), _frame0(v), _frame0(g), _frame0(be),
                             torch.from_numpy(m0).cuda(), delta=delta)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    worst = 0.0
    for b in range(wl.B):
        for h in range(wl.H):
            qh, kh, vh, gh, bh = inputs.head(wl, b, h)
            if gates is not None:
                gh = np.full_like(gh, gates[0])
                bh = np.full_like(bh, gates[1])
            ro, rs = gdn_scan_ref(qh, kh, vh, gh, bh, state_in=m0[b, h], delta=delta)
            e, _ = assert_close(to_np64(out[b, h])[None], ro, to_np64(st[b, h]), rs, TOL_BF16,
                                f"{wl.name} b{b} h{h}")
            worst = max(worst, e)
    return out, st, m0, worst


@pytest.mark.parametrize("ctas", ["2", "4"])
@pytest.mark.parametrize("S", [1, 31, 32, 33, 100, 129, 255, 500])
def test_step_shapes(monkeypatch, ctas, S):
    monkeypatch.setenv("GDN_STEP_CTAS", ctas)
    wl = inputs.Workload(f"step_s{S}", 2, 3, 64, 1, S, "bf16", 600 + S, "l2", "rollout")
    kern, P = gdn.plan(wl.B, wl.H, 1, S, 64)
    assert kern == gdn.KERNEL_STEP
    assert P == int(ctas) or (ctas == "2" and P == 4)
    _step_and_compare(wl)


@pytest.mark.parametrize("S", [880, 1350, 1408])
def test_step_large_frames(monkeypatch, S):
    monkeypatch.delenv("GDN_STEP_CTAS", raising=False)
    wl = inputs.Workload(f"step_big{S}", 1, 4, 64, 1, S, "bf16", 620 + S, "gauss", "short")
    assert gdn.plan(wl.B, wl.H, 1, S, 64) == (gdn.KERNEL_STEP, 4)
    _step_and_compare(wl)


@pytest.mark.parametrize("S", [600, 704])
def test_step_two_ctas_two_load_boxes(monkeypatch, S):
    """Two CTAs per head with more than 256 rows each: each tensor comes in two
    TMA boxes, and the read-out takes a third 128-row tile (staged in the K
    region)."""
    monkeypatch.setenv("GDN_STEP_CTAS", "2")
    wl = inputs.Workload(f"step_p2_{S}", 1, 3, 64, 1, S, "bf16", 630 + S, "l2", "rollout")
    assert gdn.plan(wl.B, wl.H, 1, S, 64) == (gdn.KERNEL_STEP, 2)
    _step_and_compare(wl)


def test_step_is_deterministic():
    """The exchanges over distributed shared memory sum the partials in a fixed
    order: the same frame stepped again, after a launch of another size in
    between, gives the same bits."""
    wl = inputs.Workload("step_repeat", 1, 32, 64, 1, 880, "bf16", 646, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    args = [_frame0(x) for x in (q, k, v, g, be)]
    o1, s1 = gdn.frame_step(*args, m0)
    small = [x[:, :3].contiguous() for x in args]
    gdn.frame_step(*small, m0[:, :3].contiguous())
    o2, s2 = gdn.frame_step(*args, m0)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_step_more_heads_than_resident_clusters():
    """60 heads: 240 CTAs in clusters of 4, more than one wave on 148 SMs."""
    wl = inputs.Workload("step_waves", 3, 20, 64, 1, 300, "bf16", 640, "lognormal", "stress")
    _step_and_compare(wl, state_scale=1.0)


def test_step_no_delta():
    wl = inputs.Workload("step_nodelta", 1, 5, 64, 1, 400, "bf16", 641, "l2", "rollout")
    _step_and_compare(wl, delta=False)


def test_step_gamma1_beta0_keeps_the_state():
    wl = inputs.Workload("step_literal", 1, 4, 64, 1, 350, "bf16", 642, "gauss", "tiny")
    out, st, m0, _ = _step_and_compare(wl, state_scale=1.0, gates=(1.0, 0.0))
    assert torch.equal(st.cpu(), torch.from_numpy(m0))


def test_step_in_place_and_null_state():
    wl = inputs.Workload("step_inplace", 2, 4, 64, 1, 880, "bf16", 643, "l2", "rollout")
    q, k, v, g, be = (_frame0(x) for x in device_workload(wl))
    m0 = torch.from_numpy(inputs.state(wl)).cuda()
    ref_o, ref_s = gdn.frame_step(q, k, v, g, be, m0.clone())
    st = m0.clone()
    o, _ = gdn.frame_step(q, k, v, g, be, st, state_out=st)
    z = torch.zeros_like(m0)
    o0, s0 = gdn.frame_step(q, k, v, g, be, None)
    oz, sz = gdn.frame_step(q, k, v, g, be, z)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o, ref_o) and torch.equal(st, ref_s)
    assert torch.equal(o0, oz) and torch.equal(s0, sz)


def test_scan_of_one_frame_is_the_step():
    """gdn_frame_scan with T = 1 takes the same kernel as gdn_frame_step."""
    wl = inputs.Workload("step_scan1", 1, 6, 64, 1, 880, "bf16", 644, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl)).cuda()
    o_scan, s_scan = gdn.frame_scan(q, k, v, g, be, m0)
    o_step, s_step = gdn.frame_step(_frame0(q), _frame0(k), _frame0(v), _frame0(g), _frame0(be), m0)
    torch.cuda.synchronize()
    assert torch.equal(o_scan[:, :, 0], o_step) and torch.equal(s_scan, s_step)


def test_step_matches_the_scan_kernel_on_a_frame(monkeypatch):
    """One frame through the step kernel and through the tensor-core scan
    kernel (GDN_STEP_CTAS=0 turns the step kernel off): the same arithmetic up
    to the fp32 summation order of K^T K and K^T V."""
    wl = inputs.Workload("step_vs_scan", 1, 8, 64, 1, 880, "bf16", 645, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    o_step, s_step = gdn.frame_scan(q, k, v, g, be, m0)
    monkeypatch.setenv("GDN_STEP_CTAS", "0")
    assert gdn.plan(wl.B, wl.H, 1, wl.S, 64) == (gdn.KERNEL_TC, 1)
    o_tc, s_tc = gdn.frame_scan(q, k, v, g, be, m0)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    e_o = float((o_step.float() - o_tc.float()).norm() / o_tc.float().norm())
    e_s = float((s_step - s_tc).norm() / s_tc.norm())
    print(f"step vs scan kernel, one frame: out {e_o:.3e}, state {e_s:.3e}")
    assert e_o <= 1e-2 and e_s <= 1e-6
