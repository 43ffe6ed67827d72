"""gdn_frame_scan_noalloc, the scan entry point for callers that must not
allocate device memory, against gdn_frame_scan, through the C ABI.

The file name sorts after every other test file, so pytest collects it last:
these tests must pass after the rest of the suite has run in the same process
(the library's per-device state already set up, the fixed scratch holding
flags and operands of earlier calls) and alone in a fresh process (the first
call on the device looks the scratch up).
"""
import ctypes

import pytest
import torch

from frame_wise_gated_scan_b200 import build, gdn, inputs
from gpu_util import TOL_BF16, assert_close, device_workload, oracle_head, to_np64

GDN_ERR_NULL = -1
GDN_ERR_SCRATCH = -8
MAX_HEADS = 32


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _scan(fn, q, k, v, g, be, state_in, state_out, out):
    B, H, T, S, D = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(_p(q), _p(k), _p(v), _p(g), _p(be), _p(state_in), _p(state_out), _p(out),
              B, H, T, S, D, stream)


def test_noalloc_limit_is_checked_on_the_host():
    build.build()
    L = gdn.lib()
    a = ctypes.c_void_p
    fake = [a(0x1000000 * (i + 1)) for i in range(8)]
    # 33 heads: one more than the fixed scratch holds; rejected before any CUDA call
    assert L.gdn_frame_scan_noalloc(*fake, 3, 11, 4, 64, 64, None) == GDN_ERR_SCRATCH
    assert L.gdn_frame_scan_noalloc(*fake, 1, MAX_HEADS + 1, 4, 64, 64, None) == GDN_ERR_SCRATCH
    assert "GDN_NOALLOC_MAX_HEADS" in gdn.status_string(GDN_ERR_SCRATCH)
    # within the limit the ordinary argument checks apply
    assert L.gdn_frame_scan_noalloc(None, *fake[1:], 1, MAX_HEADS, 4, 64, 64,
                                    None) == GDN_ERR_NULL
    # the argument checks come before the limit
    assert L.gdn_frame_scan_noalloc(None, *fake[1:], 3, 11, 4, 64, 64, None) == GDN_ERR_NULL
    # a plan without the ring (one frame: the row-split single-frame kernel) has
    # no limit; the NULL q stops the call before any launch
    assert gdn.plan(4, 50, 1, 64, 64)[0] == gdn.KERNEL_STEP
    assert L.gdn_frame_scan_noalloc(None, *fake[1:], 4, 50, 1, 64, 64, None) == GDN_ERR_NULL


@pytest.mark.gpu
@pytest.mark.parametrize("ctas", ["auto", "2", "1"])
@pytest.mark.parametrize("B,H,T,S", [(1, 4, 40, 300), (2, 16, 20, 129)])
def test_noalloc_equals_scan_over_two_calls_in_a_row(monkeypatch, ctas, B, H, T, S):
    """Two no-alloc calls back to back on one stream, on different inputs, give
    bit for bit what gdn_frame_scan gives on each: the second call must not see
    the first one's flags or operands in the shared scratch. T > 16 wraps the
    16-frame ring; (2, 16, ...) fills all 32 heads of the scratch."""
    if ctas == "auto":
        monkeypatch.delenv("GDN_TC_CTAS", raising=False)
    else:
        monkeypatch.setenv("GDN_TC_CTAS", ctas)
    kern, P = gdn.plan(B, H, T, S, 64)
    assert kern == gdn.KERNEL_TC
    if ctas != "auto":
        assert P == int(ctas)
    L = gdn.lib()
    runs = []
    for seed in (71, 72):
        wl = inputs.Workload(f"noalloc_{seed}", B, H, 64, T, S, "bf16", seed, "l2", "rollout")
        q, k, v, g, be = device_workload(wl)
        si = torch.from_numpy(inputs.state(wl, scale=0.5)).cuda()
        runs.append((wl, q, k, v, g, be, si))

    ref = []
    for wl, q, k, v, g, be, si in runs:
        out = torch.empty_like(q)
        st = torch.empty_like(si)
        assert _scan(L.gdn_frame_scan, q, k, v, g, be, si, st, out) == 0
        ref.append((out, st))
    torch.cuda.synchronize()
    assert gdn.device_status() == 0

    got = []
    for wl, q, k, v, g, be, si in runs:          # no synchronisation between the two
        out = torch.full_like(q, float("nan"))
        st = torch.full_like(si, float("nan"))
        assert _scan(L.gdn_frame_scan_noalloc, q, k, v, g, be, si, st, out) == 0
        got.append((out, st))
    torch.cuda.synchronize()
    assert gdn.device_status() == 0

    for i, ((ro, rs), (go, gs)) in enumerate(zip(ref, got)):
        assert torch.isfinite(ro).all() and torch.isfinite(rs).all()
        assert torch.equal(go, ro), f"call {i}: out differs from gdn_frame_scan"
        assert torch.equal(gs, rs), f"call {i}: state differs from gdn_frame_scan"

    # and the second call against the oracle, on one head
    wl, *_, si = runs[1]
    ro, rs = oracle_head(wl, B - 1, H - 1, state_in=si[B - 1, H - 1].cpu().numpy())
    assert_close(to_np64(got[1][0][B - 1, H - 1]), ro, to_np64(got[1][1][B - 1, H - 1]), rs,
                 TOL_BF16, "noalloc second call")


@pytest.mark.gpu
def test_noalloc_takes_nothing_from_the_stream_ordered_pool():
    """gdn_frame_scan with a clustered plan takes its ring from the device's
    default memory pool (cudaMallocAsync); the no-alloc entry point must not.
    The pool's used-memory high-water mark shows either."""
    drv = pytest.importorskip("cuda.bindings.driver")
    OK = drv.CUresult.CUDA_SUCCESS
    HIGH = drv.CUmemPool_attribute.CU_MEMPOOL_ATTR_USED_MEM_HIGH
    CUR = drv.CUmemPool_attribute.CU_MEMPOOL_ATTR_USED_MEM_CURRENT
    torch.cuda.init()
    assert drv.cuInit(0)[0] == OK
    err, dev = drv.cuDeviceGet(torch.cuda.current_device())
    assert err == OK
    err, pool = drv.cuDeviceGetDefaultMemPool(dev)
    assert err == OK

    def attr(a):
        err, v = drv.cuMemPoolGetAttribute(pool, a)
        assert err == OK
        return int(v)

    def reset_high():
        (err,) = drv.cuMemPoolSetAttribute(pool, HIGH, drv.cuuint64_t(0))
        assert err == OK

    B, H, T, S = 1, 4, 24, 256
    kern, P = gdn.plan(B, H, T, S, 64)
    assert kern == gdn.KERNEL_TC and P > 1
    wl = inputs.Workload("noalloc_pool", B, H, 64, T, S, "bf16", 73, "l2", "rollout")
    q, k, v, g, be = device_workload(wl)
    out = torch.empty_like(q)
    st = torch.empty((B, H, 64, 64), dtype=torch.float32, device=q.device)
    L = gdn.lib()
    torch.cuda.synchronize()

    base = attr(CUR)
    reset_high()
    for _ in range(2):
        assert _scan(L.gdn_frame_scan_noalloc, q, k, v, g, be, None, st, out) == 0
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert attr(HIGH) <= base, "gdn_frame_scan_noalloc took memory from the pool"

    # the probe sees the stream-ordered scratch of the ordinary entry point
    reset_high()
    assert _scan(L.gdn_frame_scan, q, k, v, g, be, None, st, out) == 0
    torch.cuda.synchronize()
    assert gdn.device_status() == 0
    assert attr(HIGH) >= base + H * 16 * 24 * 1024
