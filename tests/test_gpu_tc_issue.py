"""The D = 64 scan kernel with either issuer of the recurrence MMAs
(GDN_TC_SELF): a separate issuing thread, or the last recurrence warp done
with a frame. Only who issues the same MMAs changes, so outputs and final
states must be equal bit for bit, and match the oracle."""
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, oracle_head, to_np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P", [1, 2, 4])
@pytest.mark.parametrize("T", [1, 2, 23])
def test_recurrence_issuers_agree(monkeypatch, P, T):
    wl = inputs.Workload(f"issuer_p{P}_t{T}", 2, 3, 64, T, 200, "bf16", 800 + P + T, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    monkeypatch.setenv("GDN_TC_CTAS", str(P))
    monkeypatch.setenv("GDN_STEP_CTAS", "0")          # single frames on the scan kernel too
    res = []
    for self_issue in ("0", "1"):
        monkeypatch.setenv("GDN_TC_SELF", self_issue)
        assert gdn.plan(wl.B, wl.H, wl.T, wl.S, wl.D) == (gdn.KERNEL_TC, P)
        res.append(gdn.frame_scan(q, k, v, g, be, m0))
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
    (o0, s0), (o1, s1) = res
    assert torch.equal(o0, o1) and torch.equal(s0, s1)
    for b, h in ((0, 0), (1, 2)):
        ro, rs = oracle_head(wl, b, h, None, m0[b, h].cpu().numpy())
        assert_close(to_np64(o1[b, h]), ro, to_np64(s1[b, h]), rs, TOL_BF16, f"{wl.name} b{b} h{h}")


def test_self_issue_in_place_rollout_slice(monkeypatch):
    """Self-issued recurrence on rollout shapes (S = 880, 32 heads, 40 frames)
    with state_in == state_out, against the separate issuer."""
    wl = inputs.WORKLOADS["rollout"].with_(T=40)
    q, k, v, g, be = inputs.device_draw(wl, torch.device("cuda", 0))
    m0 = torch.randn((1, 32, 64, 64), device="cuda") * 0.1
    outs = []
    for self_issue in ("0", "1"):
        monkeypatch.setenv("GDN_TC_SELF", self_issue)
        st = m0.clone()
        o, _ = gdn.frame_scan(q, k, v, g, be, st, state_out=st)
        torch.cuda.synchronize()
        assert gdn.device_status() == 0
        outs.append((o, st))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
