"""Host-side checks of the C ABI: the library loads, exports what include/gdn.h
declares, and rejects bad arguments before touching the GPU. No compute calls."""
import ctypes
import subprocess

import pytest

from frame_wise_gated_scan_b200 import build, gdn

B, H, T, S, D = 1, 2, 3, 64, 64


@pytest.fixture(scope="module")
def L():
    build.build()
    return gdn.lib()


def test_every_declared_symbol_is_exported(L):
    names = gdn.header_symbols()
    assert set(names) >= {"gdn_frame_scan", "gdn_frame_step", "gdn_frame_scan_f32",
                          "gdn_frame_step_f32", "gdn_frame_scan_noalloc", "gdn_frame_scan_ex",
                          "gdn_frame_step_ex", "gdn_frame_scan_f32_ex", "gdn_frame_step_f32_ex",
                          "gdn_plan", "gdn_temporal_conv", "gdn_rope3d", "gdn_frame_step_rope",
                          "gdn_device_status",
                          "gdn_status_string", "gdn_version"}
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)
    # nothing else leaks out of the library
    assert {n for n in exported if not n.startswith("_")} <= set(names) | {"_init", "_fini"}


def test_version_and_strings(L):
    assert gdn.version() == 10000
    for st in range(-10, 1):
        s = gdn.status_string(st)
        assert s and s != "unknown gdn_status"
    assert gdn.status_string(-99) == "unknown gdn_status"


def _scan(L, q=0x1000, k=0x2000, v=0x3000, g=0x4000, be=0x5000, si=None, so=None, out=0x100000,
          B=B, H=H, T=T, S=S, D=D):
    p = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.gdn_frame_scan(p(q), p(k), p(v), p(g), p(be), p(si), p(so), p(out), B, H, T, S, D,
                            None)


def test_argument_errors_need_no_gpu(L):
    assert _scan(L, q=None) == -1
    assert _scan(L, out=None) == -1
    assert _scan(L, g=None) == -1
    assert _scan(L, D=48) == -3
    assert _scan(L, D=256) == -3
    assert _scan(L, T=0) == -2
    assert _scan(L, S=0) == -2
    assert _scan(L, B=-1) == -2
    assert _scan(L, q=0x1008) == -4                 # 8-byte aligned only
    assert _scan(L, g=0x4002) == -4
    assert _scan(L, si=0x9000 + 4) == -4
    assert _scan(L, out=0x1000 + 64) == -7          # out overlaps q
    n = B * H * T * S * D * 2
    assert _scan(L, q=0x10000000, k=0x20000000, v=0x30000000,
                 out=0x40000000, si=0x40000000 + n - 16) == -7   # out overlaps state_in
    # state_in == state_out is allowed (in-place); partial overlap is not
    assert _scan(L, q=0x10000000, k=0x20000000, v=0x30000000, out=0x40000000,
                 si=0x50000000, so=0x50000000 + 16) == -7


def test_step_and_f32_entry_points_validate(L):
    p = ctypes.c_void_p
    assert L.gdn_frame_step(None, p(0x2000), p(0x3000), p(0x4000), p(0x5000), None, None,
                            p(0x6000), 1, 1, 8, 64, None) == -1
    assert L.gdn_frame_step_f32(p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), None,
                                None, p(0x7000), 1, 1, 8, 96, None) == -3


def test_flags_are_checked_on_the_host(L):
    p = ctypes.c_void_p
    args = [p(0x1000), p(0x2000), p(0x3000), p(0x4000), p(0x5000), None, None, p(0x100000)]
    assert L.gdn_frame_scan_ex(*args, 1, 2, 3, 64, 64, 2, None) == -9      # unknown bit
    assert L.gdn_frame_scan_ex(*args, 1, 2, 3, 64, 64, 0x80000000, None) == -9
    assert L.gdn_frame_step_ex(*args, 1, 2, 64, 64, 4, None) == -9
    assert L.gdn_frame_scan_f32_ex(*args, 1, 2, 3, 64, 64, 3, None) == -9
    assert L.gdn_frame_step_f32_ex(*args, 1, 2, 64, 64, 8, None) == -9
    # the ordinary checks still come first
    assert L.gdn_frame_scan_ex(None, *args[1:], 1, 2, 3, 64, 64, 1, None) == -1
    assert L.gdn_frame_scan_ex(*args, 1, 2, 3, 64, 48, 1, None) == -3
    assert "GDN_FLAG_NO_DELTA" in gdn.status_string(-9)


def test_plan_is_host_logic(L):
    kern, ctas = gdn.plan(1, 32, 961, 880, 64)
    assert kern in (gdn.KERNEL_SIMT, gdn.KERNEL_TC) and ctas >= 1
    kern, ctas = gdn.plan(1, 2, 8, 64, 32)
    assert kern == gdn.KERNEL_SIMT and ctas == 1
    with pytest.raises(gdn.GdnError):
        gdn.plan(1, 1, 1, 1, 40)


def test_conv_rope_and_fused_step_validate_on_the_host(L):
    p = ctypes.c_void_p
    x, y, w = p(0x10000000), p(0x20000000), p(0x30000000)
    conv = lambda *a, **kw: L.gdn_temporal_conv(*a)
    assert L.gdn_temporal_conv(x, w, None, None, None, y, 1, 4, 3, 12, 2, None) == -2   # C % 8
    assert L.gdn_temporal_conv(x, w, None, None, None, y, 1, 4, 3, 16, 0, None) == -2   # F = 0
    assert L.gdn_temporal_conv(None, w, None, None, None, y, 1, 4, 3, 16, 2, None) == -1
    assert L.gdn_temporal_conv(p(0x10000008), w, None, None, None, y, 1, 4, 3, 16, 2, None) == -4
    assert L.gdn_temporal_conv(x, w, None, None, None, p(0x10000000 + 64), 1, 4, 3, 16, 2,
                               None) == -7                                           # y overlaps x
    assert L.gdn_temporal_conv(x, w, None, p(0x40000000), p(0x40000000 + 16), y, 1, 4, 3, 16, 2,
                               None) == -7                                           # caches overlap
    assert L.gdn_rope3d(x, y, 1, 1, 2, 8, 64, 0, 0, None) == -2                       # grid_w = 0
    assert L.gdn_rope3d(x, y, 1, 1, 2, 8, 64, 4, -1, None) == -2                      # t0 < 0
    assert L.gdn_rope3d(x, y, 1, 1, 2, 8, 48, 4, 0, None) == -3
    assert L.gdn_rope3d(None, y, 1, 1, 2, 8, 64, 4, 0, None) == -1
    assert L.gdn_rope3d(x, p(0x10000000 + 32), 1, 1, 2, 8, 64, 4, 0, None) == -7
    args = [p(0x1000000), p(0x2000000), p(0x3000000), p(0x4000000), p(0x5000000), None, None,
            p(0x6000000)]
    assert L.gdn_frame_step_rope(*args, 1, 2, 64, 128, 8, 0, 0, None) == -10          # D = 128
    assert L.gdn_frame_step_rope(*args, 1, 2, 1409, 64, 8, 0, 0, None) == -10         # S too large
    assert L.gdn_frame_step_rope(*args, 1, 2, 64, 64, 0, 0, 0, None) == -2            # grid_w = 0
    assert L.gdn_frame_step_rope(*args, 1, 2, 64, 64, 8, 0, 2, None) == -9            # flags
