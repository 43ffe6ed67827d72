"""Failure detection on the GPU without a fault: device-side waits that run out.

Every wait in the cluster kernels is bounded. The GDN_DEBUG build of the
library (libgdn_debug.so) reads the bound of role waits from
GDN_DEBUG_WAIT_NS (drains of copies and MMAs in flight keep their full 1 s
bound). With a bound of 0, some wait of every kernel runs out: the kernel
must stop, drain, return, and record GDN_ERR_TIMEOUT for gdn_device_status(),
leaving the context usable, so that the next call with the normal bound
matches the float64 oracle. Each case runs in its own process, on the debug
library only.
"""
import json
import os
import subprocess
import sys

import pytest

from frame_wise_gated_scan_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GDN_ERR_TIMEOUT = -6

CHILD = r"""
import ctypes, json, os, sys
import numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, os.path.join(ROOT, "tests"))
from frame_wise_gated_scan_b200 import inputs
from oracle import gdn_scan_ref, rel_frobenius
L = ctypes.CDLL(LIB)
vp, i = ctypes.c_void_p, ctypes.c_int
L.gdn_frame_scan.argtypes = [vp] * 8 + [i] * 5 + [vp]
L.gdn_frame_scan.restype = i
L.gdn_device_status.restype = i
L.gdn_plan.argtypes = [i] * 5 + [ctypes.POINTER(i)] * 2
B, H, T, S, D = SIZES
wl = inputs.Workload("timeout", B, H, D, T, S, "bf16", 990 + D + T, "l2", "rollout")
q, k, v, g, be = inputs.full(wl)
dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(dt)
dq, dk, dv = (dev(x, torch.bfloat16) for x in (q, k, v))
dg, db = dev(g, torch.float32), dev(be, torch.float32)
out = torch.empty_like(dq)
st = torch.empty((B, H, D, D), device="cuda")
kern, ctas = i(), i()
L.gdn_plan(B, H, T, S, D, ctypes.byref(kern), ctypes.byref(ctas))
p = lambda t: ctypes.c_void_p(t.data_ptr())
def call():
    return L.gdn_frame_scan(p(dq), p(dk), p(dv), p(dg), p(db), None, p(st), p(out), B, H, T, S, D,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
res = {"kernel": kern.value, "ctas": ctas.value}
os.environ["GDN_DEBUG_WAIT_NS"] = "0"
res["enqueue"] = call()
res["status_after_zero_budget"] = L.gdn_device_status()
os.environ["GDN_DEBUG_WAIT_NS"] = "1000000000"
res["enqueue2"] = call()
res["status_after_normal"] = L.gdn_device_status()
ro, rs = gdn_scan_ref(q, k, v, g, be)
res["out_err"] = float(np.max(rel_frobenius(out.float().cpu().numpy(), ro)))
res["state_err"] = float(np.max(rel_frobenius(st.cpu().numpy(), rs)))
print(json.dumps(res))
"""


def _debug_lib():
    path = build.build(debug=True)
    assert os.path.exists(path)
    return path


@pytest.mark.parametrize("case,sizes,env", [
    ("scan_d64_two_ctas", (1, 2, 8, 200, 64), {"GDN_TC_CTAS": "2"}),
    ("scan_d64_one_cta", (1, 2, 8, 200, 64), {"GDN_TC_CTAS": "1"}),
    ("step_row_split", (1, 2, 1, 300, 64), {}),
    ("scan_d128", (1, 2, 4, 200, 128), {}),
])
def test_wait_that_runs_out_reports_timeout_and_leaves_the_context_usable(case, sizes, env):
    lib = _debug_lib()
    code = f"ROOT = {ROOT!r}\nLIB = {lib!r}\nSIZES = {tuple(sizes)!r}\n" + CHILD
    e = dict(os.environ)
    e.pop("GDN_TC_CTAS", None)
    e.pop("GDN_STEP_CTAS", None)
    e.update(env)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=e, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    print(case, res)
    assert res["enqueue"] == 0 and res["enqueue2"] == 0
    assert res["status_after_zero_budget"] == GDN_ERR_TIMEOUT
    assert res["status_after_normal"] == 0
    assert res["out_err"] <= 2e-2 and res["state_err"] <= 2e-2
