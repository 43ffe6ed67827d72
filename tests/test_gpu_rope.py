"""3D RoPE (gdn_rope3d) against the float64 oracle, through the C ABI.

Bound, element by element: the angle p * freq is formed in fp32 (freq rounded
once from double, the product once), so it is off by at most 2^-23 p_max
radians; cos and sin, the rotation's fp32 arithmetic and the inputs' exact
bf16 values add about 2^-20 of the pair's norm; the result is rounded to bf16
(8 significant bits, 2^-8). So
    |y - y_ref| <= 2^-8 |y_ref| + (2^-23 p_max + 2^-20) * |pair|.
"""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from oracle import rope3d_ref

pytestmark = pytest.mark.gpu


def _check(y, x, grid_w, t0):
    ref = rope3d_ref(x, grid_w, t0)
    got = y.float().cpu().numpy().astype(np.float64)
    T, S = x.shape[-3], x.shape[-2]
    pmax = max(t0 + T - 1, (S - 1) // grid_w, min(S, grid_w) - 1, 1)
    pair = np.sqrt(x[..., 0::2] ** 2 + x[..., 1::2] ** 2)
    pair = np.repeat(pair, 2, axis=-1)
    bound = 2.0 ** -8 * np.abs(ref) + (2.0 ** -23 * pmax + 2.0 ** -20) * pair
    excess = float(np.max(np.abs(got - ref) - bound))
    assert excess <= 0.0, f"bound exceeded by {excess:.3e}"


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("T,S,grid_w,t0", [(1, 1, 1, 0), (3, 7, 3, 5), (2, 880, 40, 0),
                                           (2, 880, 40, 959), (1, 1350, 45, 240)])
def test_rope3d_against_oracle(D, T, S, grid_w, t0):
    wl = inputs.Workload("rope", 1, 2, D, T, S, "bf16", 900 + D + S + T, "gauss", "tiny")
    q = inputs.full(wl)[0]
    x = torch.from_numpy(q).cuda().to(torch.bfloat16)
    y = gdn.rope3d(x, grid_w, t0)
    torch.cuda.synchronize()
    _check(y, q, grid_w, t0)


def test_rope3d_in_place_equals_out_of_place():
    wl = inputs.Workload("rope_ip", 2, 3, 64, 4, 200, "bf16", 950, "l2", "rollout")
    x = torch.from_numpy(inputs.full(wl)[1]).cuda().to(torch.bfloat16)
    y = gdn.rope3d(x, 20, 7)
    z = x.clone()
    gdn.rope3d(z, 20, 7, out=z)
    torch.cuda.synchronize()
    assert torch.equal(y, z)


def test_rope3d_bad_arguments():
    x = torch.zeros((1, 1, 1, 4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.rope3d(x, 0)
    assert ei.value.status == -2
    with pytest.raises(gdn.GdnError) as ei:
        gdn.rope3d(x, 4, -1)
    assert ei.value.status == -2
    x = torch.zeros((1, 1, 1, 4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.rope3d(x, 4)
    assert ei.value.status == -3


# ---- 3D RoPE fused into the single-frame step (gdn_frame_step_rope) ----

@pytest.mark.parametrize("S,grid_w,frame", [(880, 40, 0), (880, 40, 500), (300, 20, 7), (1350, 45, 240)])
def test_fused_rope_step_equals_rope_then_step(S, grid_w, frame):
    """Turning q and k in shared memory gives bit for bit what rotating them in
    HBM first and then stepping gives."""
    wl = inputs.Workload("rope_step", 1, 4, 64, 1, S, "bf16", 960 + S + frame, "l2", "rollout")
    q, k, v, g, be = (torch.from_numpy(a).cuda() for a in inputs.full(wl))
    q, k, v = (x.to(torch.bfloat16)[:, :, 0].contiguous() for x in (q, k, v))
    g, be = g[:, :, 0].contiguous(), be[:, :, 0].contiguous()
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    of, sf = gdn.frame_step(q, k, v, g, be, m0, rope=(grid_w, frame))
    qr = gdn.rope3d(q[:, :, None].contiguous(), grid_w, frame)[:, :, 0].contiguous()
    kr = gdn.rope3d(k[:, :, None].contiguous(), grid_w, frame)[:, :, 0].contiguous()
    ou, su = gdn.frame_step(qr, kr, v, g, be, m0)
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert torch.equal(of, ou) and torch.equal(sf, su)


def test_fused_rope_step_against_oracle():
    """Oracle side: rotate in float64, then the GDN update of one frame."""
    from oracle import gdn_scan_ref, rel_frobenius
    wl = inputs.Workload("rope_step_oracle", 1, 3, 64, 1, 880, "bf16", 970, "l2", "rollout")
    qn, kn, vn, gn, bn = inputs.full(wl)
    m0 = inputs.state(wl, scale=0.5)
    dev = lambda a, dt: torch.from_numpy(a).cuda().to(dt)
    o, st = gdn.frame_step(dev(qn[:, :, 0], torch.bfloat16), dev(kn[:, :, 0], torch.bfloat16),
                           dev(vn[:, :, 0], torch.bfloat16), dev(gn[:, :, 0], torch.float32),
                           dev(bn[:, :, 0], torch.float32), dev(m0, torch.float32), rope=(40, 123))
    torch.cuda.synchronize()
    qr, kr = rope3d_ref(qn, 40, 123), rope3d_ref(kn, 40, 123)
    ro, rs = gdn_scan_ref(qr, kr, vn, gn, bn, state_in=m0)
    e_o = float(np.max(rel_frobenius(o.float().cpu().numpy()[:, :, None], ro)))
    e_s = float(np.max(rel_frobenius(st.cpu().numpy(), rs)))
    assert e_o <= 2e-2 and e_s <= 2e-2, (e_o, e_s)


def test_fused_rope_step_unsupported_sizes():
    x = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    g = torch.ones((1, 1), device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.frame_step(x, x.clone(), x.clone(), g, g.clone(), rope=(8, 0))
    assert ei.value.status == -10
