"""Host logic that needs no GPU: which kernel and cluster size a call gets, and
that the product path fails loudly, with no fallback, when the library is
missing."""
import os
import subprocess
import sys

import pytest
import torch

from frame_wise_gated_scan_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TC, SIMT, STEP = gdn.KERNEL_TC, gdn.KERNEL_SIMT, gdn.KERNEL_STEP


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="with a device the thresholds come from its SM count")
def test_plan_without_a_device(monkeypatch):
    monkeypatch.delenv("GDN_TC_CTAS", raising=False)
    # 148 SMs assumed: 33 clusters of 4 (whole GPCs), 74 of 2 fit at once
    assert gdn.plan(1, 32, 961, 880, 64) == (TC, 4)
    assert gdn.plan(1, 33, 2, 64, 64) == (TC, 4)
    assert gdn.plan(1, 34, 2, 64, 64) == (TC, 2)
    assert gdn.plan(2, 37, 2, 64, 64) == (TC, 2)
    assert gdn.plan(1, 75, 2, 64, 64) == (TC, 1)


def test_plan_rules_that_hold_on_any_machine(monkeypatch):
    monkeypatch.delenv("GDN_TC_CTAS", raising=False)
    monkeypatch.delenv("GDN_STEP_CTAS", raising=False)
    # a single frame: the row-split kernel, 4 CTAs per head share the rows
    assert gdn.plan(1, 32, 1, 880, 64) == (STEP, 4)
    assert gdn.plan(4, 16, 1, 1408, 64) == (STEP, 4)       # 352 rows per CTA, its limit
    assert gdn.plan(1, 32, 1, 1409, 64) == (TC, 1)         # more rows: one CTA streams them
    assert gdn.plan(1, 2, 1, 1, 64) == (STEP, 4)
    assert gdn.plan(1, 2, 1, 64, 128) == (TC, 2)           # D = 128: producer + reader CTAs
    monkeypatch.setenv("GDN_STEP_CTAS", "2")
    assert gdn.plan(1, 32, 1, 500, 64) == (STEP, 2)
    assert gdn.plan(1, 32, 1, 880, 64) == (STEP, 4)        # 440 rows per CTA would not fit
    monkeypatch.setenv("GDN_STEP_CTAS", "0")               # off: the scan kernel, one CTA
    assert gdn.plan(1, 32, 1, 880, 64) == (TC, 1)
    monkeypatch.delenv("GDN_STEP_CTAS")
    assert gdn.plan(4, 16, 241, 1350, 128) == (TC, 2)      # D = 128: producer + reader CTAs
    assert gdn.plan(1, 2, 8, 64, 32) == (SIMT, 1)          # D = 32
    for forced in ("1", "2", "4"):
        monkeypatch.setenv("GDN_TC_CTAS", forced)
        assert gdn.plan(1, 32, 961, 880, 64) == (TC, int(forced))
    monkeypatch.setenv("GDN_TC_CTAS", "3")                 # not a cluster size it builds
    assert gdn.plan(1, 32, 2, 880, 64) == (TC, 4) or gdn.plan(1, 32, 2, 880, 64)[0] == TC
    with pytest.raises(gdn.GdnError):
        gdn.plan(1, 32, 961, 880, 48)


def test_impl_override_routes_to_cuda_cores():
    env = dict(os.environ, GDN_IMPL="simt")
    env.pop("GDN_TC_CTAS", None)
    code = ("from frame_wise_gated_scan_b200 import gdn; "
            "print(gdn.plan(1, 32, 961, 880, 64))")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                         text=True, check=True).stdout.strip()
    assert out == f"({SIMT}, 1)"


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libgdn.so"))
    with pytest.raises(RuntimeError, match="not built"):
        gdn.lib()
    with pytest.raises(RuntimeError, match="not built"):
        gdn.plan(1, 32, 961, 880, 64)
