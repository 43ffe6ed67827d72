"""Builds libgdn.so in-tree with nvcc for sm_100a.

    python -m frame_wise_gated_scan_b200.build [--debug]

The shared library lands next to this file; the Python binding loads it from
there and nowhere else.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgdn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


DEBUG_LIB = os.path.join(PKG, "libgdn_debug.so")


def build(debug: bool = False, verbose: bool = False, force: bool = False,
          trace_out: str | None = None, out: str | None = None) -> str:
    """Builds libgdn.so. With trace_out, builds instead a pipeline-trace variant
    (GDN_TRACE: per-frame event timestamps of head 0, read with gdn_trace_copy)
    at that path; the library the binding loads is left untouched. With
    debug=True, builds the GDN_DEBUG variant (device-wait budget read from
    GDN_DEBUG_WAIT_NS) at `out`, by default libgdn_debug.so."""
    if debug and out is None:
        out = DEBUG_LIB
    out = trace_out or out or LIB
    if not force and not trace_out and not needs_build(out):
        return out
    cmd = [nvcc(), *ARCH, "-std=c++17", "-O3", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
           "-I", INCLUDE, "-I", CSRC, "-o", out, *sources(), "-lcudart_static", "-ldl", "-lrt",
           "-lpthread"]
    if debug:
        cmd.insert(1, "-DGDN_DEBUG=1")
    if trace_out:
        cmd.insert(1, "-DGDN_TRACE=1")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libgdn.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    return out


if __name__ == "__main__":
    trace = None
    if "--trace-out" in sys.argv:
        trace = sys.argv[sys.argv.index("--trace-out") + 1]
    print(build(debug="--debug" in sys.argv, verbose="-v" in sys.argv, force=True, trace_out=trace))
