"""Chunk-causal streaming through the device-side frame queue
(gdn_frame_stream): one persistent launch, frames posted one at a time.

The streaming kernel runs the arithmetic of the row-split single-frame kernel
and keeps the state on chip between frames; the state it carries (fp32 rows
plus their bf16 copy for the next product) is what a chain of gdn_frame_step
calls writes to and reads back from HBM. So its outputs and final state must
equal the step chain's bit for bit, and match the oracle within 2e-2.
"""
import numpy as np
import pytest
import torch

from frame_wise_gated_scan_b200 import gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, oracle_head, to_np64

pytestmark = pytest.mark.gpu


def _rings(wl):
    """The workload as rings [T, B, H, ...] (frame n in slot n)."""
    q, k, v, g, be = device_workload(wl)
    ring = lambda x: x.permute(2, 0, 1, *range(3, x.dim())).contiguous()
    return ring(q), ring(k), ring(v), ring(g), ring(be)


def _step_chain(qr, kr, vr, gr, br, m0):
    st = m0.clone()
    outs = []
    for t in range(qr.shape[0]):
        o, _ = gdn.frame_step(qr[t], kr[t], vr[t], gr[t], br[t], st, state_out=st)
        outs.append(o)
    return torch.stack(outs), st


def test_stream_equals_step_chain_one_frame_at_a_time():
    wl = inputs.Workload("stream", 1, 6, 64, 12, 880, "bf16", 1100, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    ref_o, ref_s = _step_chain(qr, kr, vr, gr, br, m0)
    torch.cuda.synchronize()
    fs = gdn.FrameStream(qr, kr, vr, gr, br, state_in=m0)
    for n in range(wl.T):          # nothing but posts and polls while the launch runs
        fs.post()
        fs.wait(n + 1)
    st = fs.close()
    assert torch.equal(fs.out, ref_o) and torch.equal(st, ref_s)
    # and against the oracle on two heads
    for h in (0, 5):
        ro, rs = oracle_head(wl, 0, h, state_in=m0[0, h].cpu().numpy())
        assert_close(to_np64(fs.out[:, 0, h]), ro, to_np64(st[0, h]), rs, TOL_BF16, f"stream h{h}")


def test_stream_all_frames_posted_at_once_and_no_delta():
    wl = inputs.Workload("stream_batch", 2, 3, 64, 7, 300, "bf16", 1101, "gauss", "short")
    qr, kr, vr, gr, br = _rings(wl)
    z = torch.zeros((wl.B, wl.H, 64, 64), device="cuda")
    st = z.clone()
    outs = []
    for t in range(wl.T):
        o, _ = gdn.frame_step(qr[t], kr[t], vr[t], gr[t], br[t], st, state_out=st, delta=False)
        outs.append(o)
    torch.cuda.synchronize()
    fs = gdn.FrameStream(qr, kr, vr, gr, br, delta=False)
    fs.post(wl.T)
    fs.wait(wl.T)
    s2 = fs.close()
    assert torch.equal(fs.out, torch.stack(outs)) and torch.equal(s2, st)


def test_stream_ring_refilled_from_host_memory():
    """Three slots for nine frames: each slot is refilled (copy engine, from
    pinned host memory) once the frame it held is done."""
    wl = inputs.Workload("stream_ring", 1, 4, 64, 9, 500, "bf16", 1102, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    ref_o, ref_s = _step_chain(qr, kr, vr, gr, br, m0)
    host = [x.cpu().pin_memory() for x in (qr, kr, vr, gr, br)]
    R = 3
    rings = [torch.empty((R,) + tuple(x.shape[1:]), dtype=x.dtype, device="cuda") for x in host]
    host_out = torch.empty(tuple(ref_o.shape), dtype=ref_o.dtype, pin_memory=True)
    out_ring = torch.empty_like(rings[0])
    copy = torch.cuda.Stream()
    with torch.cuda.stream(copy):
        for dst, src in zip(rings, host):
            dst.copy_(src[:R], non_blocking=True)
    copy.synchronize()
    torch.cuda.synchronize()
    fs = gdn.FrameStream(*rings, out=out_ring, state_in=m0)
    # while the launch runs: posts, polls, and copies between pinned host
    # memory and the pre-allocated rings on a stream of our own, nothing else
    for n in range(wl.T):
        if n >= R:
            fs.wait(n - R + 1)                       # the slot's previous frame is done
            with torch.cuda.stream(copy):
                host_out[n - R].copy_(out_ring[(n - R) % R], non_blocking=True)
                for dst, src in zip(rings, host):
                    dst[n % R].copy_(src[n], non_blocking=True)
            copy.synchronize()
        fs.post()
    fs.wait(wl.T)
    with torch.cuda.stream(copy):
        for n in range(wl.T - R, wl.T):
            host_out[n].copy_(out_ring[n % R], non_blocking=True)
    copy.synchronize()
    st = fs.close()
    assert torch.equal(host_out, ref_o.cpu()) and torch.equal(st, ref_s)


def test_stream_stop_without_frames_returns_the_state():
    wl = inputs.Workload("stream_empty", 1, 2, 64, 1, 200, "bf16", 1103, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    m0 = torch.from_numpy(inputs.state(wl)).cuda()
    fs = gdn.FrameStream(qr, kr, vr, gr, br, state_in=m0)
    assert torch.equal(fs.close(), m0)


def test_stream_idle_timeout_reports_and_leaves_the_context_usable():
    """No frame and no stop within the idle bound: the kernel stops by itself
    and the device status reports a timeout; the next call works."""
    wl = inputs.Workload("stream_idle", 1, 2, 64, 1, 200, "bf16", 1104, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    fs = gdn.FrameStream(qr, kr, vr, gr, br, idle_timeout_s=0.2)
    fs.stream.synchronize()                          # the kernel gives up after 0.2 s
    assert gdn.device_status() == -6
    o, s = gdn.frame_step(qr[0], kr[0], vr[0], gr[0], br[0])
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    ro, rs = oracle_head(wl, 0, 1)
    assert_close(to_np64(o[0, 1])[None], ro, to_np64(s[0, 1]), rs, TOL_BF16, "after idle timeout")


def test_stream_rejects_sizes_it_cannot_keep_resident():
    q = torch.zeros((2, 2, 40, 64, 64), dtype=torch.bfloat16, device="cuda")   # 80 heads
    g = torch.ones((2, 2, 40), device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.FrameStream(q, q.clone(), q.clone(), g, g.clone())
    assert ei.value.status == -10


def test_stream_with_rope_equals_rope_step_chain():
    """gdn_frame_stream_rope: frame n turned as frame t0 + n, equal bit for bit
    to gdn_frame_step_rope calls with frame_index t0, t0 + 1, ..."""
    wl = inputs.Workload("stream_rope", 1, 5, 64, 7, 880, "bf16", 1105, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    m0 = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
    grid_w, t0 = 40, 11
    st = m0.clone()
    outs = []
    for t in range(wl.T):
        o, _ = gdn.frame_step(qr[t], kr[t], vr[t], gr[t], br[t], st, state_out=st, rope=(grid_w, t0 + t))
        outs.append(o)
    ref_o = torch.stack(outs)
    torch.cuda.synchronize()
    fs = gdn.FrameStream(qr, kr, vr, gr, br, state_in=m0, rope=(grid_w, t0))
    for n in range(wl.T):
        fs.post()
        fs.wait(n + 1)
    s2 = fs.close()
    assert torch.equal(fs.out, ref_o) and torch.equal(s2, st)
    # and the rotation matters: without it the outputs differ
    assert not torch.equal(ref_o, _step_chain(qr, kr, vr, gr, br, m0)[0])


def test_stream_rope_rejects_bad_grid():
    wl = inputs.Workload("stream_rope_bad", 1, 2, 64, 1, 100, "bf16", 1106, "l2", "rollout")
    qr, kr, vr, gr, br = _rings(wl)
    with pytest.raises(gdn.GdnError) as ei:
        gdn.FrameStream(qr, kr, vr, gr, br, rope=(0, 0))
    assert ei.value.status == -2
