"""The D = 128 tensor-core kernel (a producer and a reader CTA per head)
against the float64 oracle, through the C ABI. Tolerance: relative Frobenius
error 2e-2 per frame and head for out, per head for the final state."""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, oracle_head, to_np64
from oracle import gdn_scan_ref, rel_frobenius

pytestmark = pytest.mark.gpu


def _scan(wl, state_scale=None, delta=True, gates=None):
    assert gdn.plan(wl.B, wl.H, wl.T, wl.S, wl.D) == (gdn.KERNEL_TC, 2)
    q, k, v, g, be = device_workload(wl)
    if gates is not None:
        g = torch.full_like(g, gates[0])
        be = torch.full_like(be, gates[1])
    m0 = None if state_scale is None else inputs.state(wl, scale=state_scale)
    out, st = gdn.frame_scan(q, k, v, g, be, None if m0 is None else torch.from_numpy(m0).cuda(),
                             delta=delta)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    return out, st, m0, g, be


def _compare(wl, out, st, m0, heads, delta=True, gates=None):
    worst = (0.0, 0.0)
    for b, h in heads:
        qh, kh, vh, gh, bh = inputs.head(wl, b, h)
        if gates is not None:
            gh, bh = np.full_like(gh, gates[0]), np.full_like(bh, gates[1])
        ro, rs = gdn_scan_ref(qh, kh, vh, gh, bh, state_in=None if m0 is None else m0[b, h],
                              delta=delta)
        eo, es = assert_close(to_np64(out[b, h]), ro, to_np64(st[b, h]), rs, TOL_BF16,
                              f"{wl.name} b{b} h{h}")
        worst = (max(worst[0], eo), max(worst[1], es))
    return worst


@pytest.mark.parametrize("T", [1, 3])
@pytest.mark.parametrize("S", [1, 6, 63, 64, 65, 127, 128, 129, 300])
def test_d128_shapes(S, T):
    wl = inputs.Workload(f"d128_s{S}_t{T}", 1, 3, 128, T, S, "bf16", 800 + S + T, "gauss", "tiny")
    out, st, m0, *_ = _scan(wl, state_scale=0.5)
    _compare(wl, out, st, m0, [(0, h) for h in range(3)])


def test_d128_frames_and_state():
    wl = inputs.Workload("d128_frames", 2, 3, 128, 17, 1350, "bf16", 820, "l2", "rollout")
    out, st, m0, *_ = _scan(wl, state_scale=0.5)
    _compare(wl, out, st, m0, [(0, 0), (1, 2)])


def test_d128_more_heads_than_resident_clusters():
    """80 heads: 160 CTAs in clusters of two, more than one wave on 148 SMs."""
    wl = inputs.Workload("d128_waves", 4, 20, 128, 4, 200, "bf16", 821, "gauss", "short")
    out, st, m0, *_ = _scan(wl)
    _compare(wl, out, st, m0, [(0, 0), (2, 7), (3, 19)])


def test_d128_no_delta():
    wl = inputs.Workload("d128_nodelta", 1, 3, 128, 9, 257, "bf16", 822, "l2", "rollout")
    out, st, m0, *_ = _scan(wl, state_scale=0.5, delta=False)
    _compare(wl, out, st, m0, [(0, 0), (0, 2)], delta=False)


def test_d128_gamma1_beta0_keeps_the_state():
    wl = inputs.Workload("d128_literal", 1, 2, 128, 12, 300, "bf16", 823, "lognormal", "stress")
    out, st, m0, *_ = _scan(wl, state_scale=1.0, gates=(1.0, 0.0))
    assert torch.equal(st.cpu(), torch.from_numpy(m0))
    _compare(wl, out, st, m0, [(0, 0), (0, 1)], gates=(1.0, 0.0))


def test_d128_beta0_decays_by_gamma_products():
    wl = inputs.Workload("d128_decay", 1, 2, 128, 40, 200, "bf16", 824, "l2", "rollout")
    q, k, v, g, _ = device_workload(wl)
    be = torch.zeros_like(g)
    m0 = inputs.state(wl)
    out, st = gdn.frame_scan(q, k, v, g, be, torch.from_numpy(m0).cuda())
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    gam = g.double().cpu().numpy()
    for h in range(2):
        expect = np.prod(gam[0, h]) * m0[0, h].astype(np.float64)
        e = float(np.max(rel_frobenius(to_np64(st[0, h]), expect)))
        assert e <= wl.T * 2.0 ** -23, f"beta = 0 decay h{h}: {e:.3e}"


def test_d128_in_place_and_null_state():
    wl = inputs.Workload("d128_inplace", 1, 4, 128, 5, 200, "bf16", 825, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl)).cuda()
    ref_o, ref_s = gdn.frame_scan(q, k, v, g, be, m0.clone())
    st = m0.clone()
    o, _ = gdn.frame_scan(q, k, v, g, be, st, state_out=st)
    o0, s0 = gdn.frame_scan(q, k, v, g, be, None)
    oz, sz = gdn.frame_scan(q, k, v, g, be, torch.zeros_like(m0))
    o3, s3 = gdn.frame_scan(q, k, v, g, be, None, want_state=False)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(o, ref_o) and torch.equal(st, ref_s)
    assert torch.equal(o0, oz) and torch.equal(s0, sz) and torch.equal(o0, o3) and s3 is None


def test_d128_stress_recipe_sampled():
    """The stress recipe (log-normal key norms, gamma ~ U(.99,1), beta = 1) on a
    few heads over 60 frames: near-unit decay on the tensor-core path."""
    wl = inputs.Workload("d128_stress", 2, 4, 128, 60, 1350, "bf16", 5, "lognormal", "stress")
    out, st, m0, *_ = _scan(wl)
    worst = _compare(wl, out, st, m0, [(0, 0), (1, 3)])
    print(f"stress recipe D=128, 60 frames: out {worst[0]:.3e}, state {worst[1]:.3e}")
