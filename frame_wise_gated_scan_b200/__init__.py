"""libgdn: the frame-wise Gated DeltaNet scan on B200, behind a C ABI (include/gdn.h).

Python users call frame_scan / frame_step / frame_scan_host (and
frame_scan_noalloc, for callers that must not allocate device memory) from
frame_wise_gated_scan_b200.gdn; the library is built in-tree by
frame_wise_gated_scan_b200.build.
"""
from .gdn import (FLAG_NO_DELTA, GdnError, KERNEL_SIMT, KERNEL_TC, device_status, frame_scan,
                  frame_scan_host,
                  frame_scan_noalloc, frame_step, plan, version)

__all__ = ["FLAG_NO_DELTA", "GdnError", "KERNEL_SIMT", "KERNEL_TC", "device_status", "frame_scan",
           "frame_scan_host", "frame_scan_noalloc", "frame_step", "plan", "version"]
