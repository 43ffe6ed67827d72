"""Python binding of libgdn (include/gdn.h): argument marshalling only.

Every step of the recurrence runs in the library's CUDA kernels. This module
checks tensors, allocates outputs with torch (device memory is the caller's
side of the ABI), passes raw pointers and the current CUDA stream, and turns
a negative status into GdnError. There is no fallback: without the built
library every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "gdn.h")

KERNEL_SIMT = 1
KERNEL_TC = 2
KERNEL_STEP = 3
FLAG_NO_DELTA = 1     # GDN_FLAG_NO_DELTA: R = V, the decayed cumulative (block KV cache) form

_lib = None


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def header_symbols() -> list[str]:
    """Names of the functions include/gdn.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)


def lib() -> ctypes.CDLL:
    """The in-tree libgdn.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libgdn.so not built at {LIB_PATH}; run "
                               "python -m frame_wise_gated_scan_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, i = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        scan_args = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, i, vp]
        step_args = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, vp]
        for name, args in (("gdn_frame_scan", scan_args), ("gdn_frame_scan_f32", scan_args),
                           ("gdn_frame_scan_noalloc", scan_args),
                           ("gdn_frame_step", step_args), ("gdn_frame_step_f32", step_args)):
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = i
        u = ctypes.c_uint
        for name, args in (("gdn_frame_scan_ex", scan_args[:-1] + [u, vp]),
                           ("gdn_frame_scan_f32_ex", scan_args[:-1] + [u, vp]),
                           ("gdn_frame_step_ex", step_args[:-1] + [u, vp]),
                           ("gdn_frame_step_f32_ex", step_args[:-1] + [u, vp])):
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = i
        L.gdn_temporal_conv.argtypes = [vp, fp, fp, vp, vp, vp, i, i, i, i, i, vp]
        L.gdn_temporal_conv.restype = i
        L.gdn_frame_step_rope.argtypes = step_args[:-1] + [i, i, u, vp]
        L.gdn_frame_step_rope.restype = i
        ull = ctypes.c_ulonglong
        L.gdn_frame_stream.argtypes = step_args[:-1] + [i, vp, vp, vp, ull, u, vp]
        L.gdn_frame_stream.restype = i
        L.gdn_frame_stream_rope.argtypes = step_args[:-1] + [i, vp, vp, vp, ull, i, i, u, vp]
        L.gdn_frame_stream_rope.restype = i
        L.gdn_rope3d.argtypes = [vp, vp, i, i, i, i, i, i, i, vp]
        L.gdn_rope3d.restype = i
        L.gdn_plan.argtypes = [i, i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(i)]
        L.gdn_plan.restype = i
        L.gdn_device_status.argtypes = []
        L.gdn_device_status.restype = i
        L.gdn_status_string.argtypes = [i]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_version.argtypes = []
        L.gdn_version.restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def version() -> int:
    return lib().gdn_version()


def plan(B: int, H: int, T: int, S: int, D: int) -> tuple[int, int]:
    """(kernel id, CTAs per head) a bf16 call with these sizes would use."""
    k, c = ctypes.c_int(), ctypes.c_int()
    st = lib().gdn_plan(B, H, T, S, D, ctypes.byref(k), ctypes.byref(c))
    if st != 0:
        raise GdnError(st, "gdn_plan")
    return k.value, c.value


def device_status() -> int:
    """Synchronizes and returns the library's device status (0 = no wait ran out)."""
    return lib().gdn_device_status()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def step_args(q, k, v, gamma, beta, state_in, state_out, out, stream=None):
    """The raw argument list of gdn_frame_step for these tensors, for callers
    that issue many calls on the same buffers: lib().gdn_frame_step(*args)
    then costs one ctypes call. The tensors are checked once, here."""
    frame_step(q, k, v, gamma, beta, state_in, out=out, state_out=state_out)   # validates
    B, H, S, D = q.shape
    stream = stream or torch.cuda.current_stream(q.device)
    return [_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(state_out),
            _ptr(out), B, H, S, D, ctypes.c_void_p(stream.cuda_stream)]


def _check(t, name, dtype, shape, device):
    if t.dtype is dtype and t.shape == shape and t.is_contiguous() and t.device == device:
        return                                   # the common case, in one test
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _call(step: bool, q, k, v, gamma, beta, state_in, out, state_out, want_state,
          noalloc=False, flags=0, rope=None):
    if q.dim() != (4 if step else 5):
        raise ValueError("q must be [B,H,S,D] for a step, [B,H,T,S,D] for a scan")
    device = q.device
    if device.type != "cuda":
        raise ValueError("tensors must be CUDA tensors (use frame_scan_host for host buffers)")
    dt = q.dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bfloat16 or float32")
    if step:
        B, H, S, D = q.shape
        T = 1
        gshape = (B, H)
    else:
        B, H, T, S, D = q.shape
        gshape = (B, H, T)
    for name, t in (("k", k), ("v", v)):
        _check(t, name, dt, q.shape, device)
    _check(gamma, "gamma", torch.float32, gshape, device)
    _check(beta, "beta", torch.float32, gshape, device)
    if state_in is not None:
        _check(state_in, "state_in", torch.float32, (B, H, D, D), device)
    if out is None:
        out = torch.empty_like(q)
    else:
        _check(out, "out", dt, q.shape, device)
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=device)
    elif state_out is not None:
        _check(state_out, "state_out", torch.float32, (B, H, D, D), device)
    L = lib()
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in),
            _ptr(state_out), _ptr(out), B, H]
    if not step:
        args.append(T)
    args += [S, D]
    if rope is not None:
        if not step or dt != torch.bfloat16:
            raise ValueError("the fused 3D RoPE is a bf16 single-frame option")
        args += [int(rope[0]), int(rope[1]), flags]
    elif flags:
        args.append(flags)
    args.append(_stream_handle(device))
    bf16 = dt == torch.bfloat16
    if rope is not None:
        fn = L.gdn_frame_step_rope
    elif flags:
        if step:
            fn = L.gdn_frame_step_ex if bf16 else L.gdn_frame_step_f32_ex
        else:
            fn = L.gdn_frame_scan_ex if bf16 else L.gdn_frame_scan_f32_ex
    elif noalloc:
        fn = L.gdn_frame_scan_noalloc
    elif step:
        fn = L.gdn_frame_step if dt == torch.bfloat16 else L.gdn_frame_step_f32
    else:
        fn = L.gdn_frame_scan if dt == torch.bfloat16 else L.gdn_frame_scan_f32
    if device.index == torch.cuda.current_device():
        st = fn(*args)
    else:
        with torch.cuda.device(device):
            st = fn(*args)
    if st != 0:
        raise GdnError(st, fn.__name__)
    return out, state_out


def frame_scan(q, k, v, gamma, beta, state_in=None, *, out=None, state_out=None,
               want_state=True, delta=True):
    """T frames per head. q, k, v: [B,H,T,S,D] bf16 or fp32 CUDA tensors;
    gamma, beta: [B,H,T] fp32; state_in: [B,H,D,D] fp32 or None (zero).
    delta=False drops the delta-rule correction (GDN_FLAG_NO_DELTA: R = V).
    Returns (out, state_out); state_out is None if want_state is False and
    none was given."""
    return _call(False, q, k, v, gamma, beta, state_in, out, state_out, want_state,
                 flags=0 if delta else FLAG_NO_DELTA)


def frame_scan_noalloc(q, k, v, gamma, beta, state_in=None, *, out, state_out=None):
    """frame_scan through gdn_frame_scan_noalloc, for callers that must not
    allocate device memory: bf16 only, B*H <= 32, and out (plus state_out, if
    the final state is wanted) supplied by the caller, so nothing is allocated
    here either. Calls on one device must not overlap on the GPU: they share
    the library's fixed scratch."""
    if q.dtype != torch.bfloat16:
        raise TypeError("frame_scan_noalloc takes bfloat16 q, k, v")
    if q.dim() != 5:
        raise ValueError("q must be [B,H,T,S,D]")
    return _call(False, q, k, v, gamma, beta, state_in, out, state_out, False, noalloc=True)


def frame_step(q, k, v, gamma, beta, state_in=None, *, out=None, state_out=None,
               want_state=True, delta=True, rope=None):
    """One frame per head (chunk-causal rollout). q, k, v: [B,H,S,D];
    gamma, beta: [B,H]. state_out may be state_in (in-place carry).
    delta=False as in frame_scan. rope=(grid_w, frame_index) turns q and k by
    3D RoPE inside the kernel first (gdn_frame_step_rope)."""
    return _call(True, q, k, v, gamma, beta, state_in, out, state_out, want_state,
                 flags=0 if delta else FLAG_NO_DELTA, rope=rope)


def temporal_conv(x, w, bias=None, cache_in=None, *, frames_per_block=None, y=None,
                  cache_out=None, want_cache=True):
    """Causal temporal convolution with a carried last-frame cache
    (gdn_temporal_conv). x: [B,T,S,C] bf16 CUDA tensor; w: [C,3] fp32 taps for
    the previous, current and next frame; bias: [C] fp32 or None; cache_in:
    [B,S,C] bf16 (the previous call's last frame) or None for zeros;
    frames_per_block: block length (None: the whole call is one block).
    cache_out may be cache_in. Returns (y, cache_out); cache_out is None if
    want_cache is False and none was given."""
    if x.dim() != 4 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a [B,T,S,C] bfloat16 tensor")
    device = x.device
    if device.type != "cuda":
        raise ValueError("x must be a CUDA tensor")
    B, T, S, C = x.shape
    _check(x, "x", torch.bfloat16, (B, T, S, C), device)
    _check(w, "w", torch.float32, (C, 3), device)
    if bias is not None:
        _check(bias, "bias", torch.float32, (C,), device)
    if cache_in is not None:
        _check(cache_in, "cache_in", torch.bfloat16, (B, S, C), device)
    if y is None:
        y = torch.empty_like(x)
    else:
        _check(y, "y", torch.bfloat16, (B, T, S, C), device)
    if cache_out is None and want_cache:
        cache_out = torch.empty((B, S, C), dtype=torch.bfloat16, device=device)
    elif cache_out is not None:
        _check(cache_out, "cache_out", torch.bfloat16, (B, S, C), device)
    F = T if frames_per_block is None else int(frames_per_block)
    L = lib()
    with torch.cuda.device(device):
        st = L.gdn_temporal_conv(_ptr(x), _ptr(w), _ptr(bias), _ptr(cache_in), _ptr(cache_out),
                                 _ptr(y), B, T, S, C, F, _stream_handle(device))
    if st != 0:
        raise GdnError(st, "gdn_temporal_conv")
    return y, cache_out


def rope3d(x, grid_w, t0=0, *, out=None):
    """3D RoPE of queries or keys (gdn_rope3d): x [B,H,T,S,D] bf16 CUDA tensor,
    token r of a frame at grid row r // grid_w, column r % grid_w, frame index
    t0 + tau. out may be x (in place). Returns the rotated tensor."""
    if x.dim() != 5 or x.dtype != torch.bfloat16 or x.device.type != "cuda":
        raise ValueError("x must be a [B,H,T,S,D] bfloat16 CUDA tensor")
    B, H, T, S, D = x.shape
    _check(x, "x", torch.bfloat16, x.shape, x.device)
    if out is None:
        out = torch.empty_like(x)
    else:
        _check(out, "out", torch.bfloat16, x.shape, x.device)
    with torch.cuda.device(x.device):
        st = lib().gdn_rope3d(_ptr(x), _ptr(out), B, H, T, S, D, int(grid_w), int(t0),
                              _stream_handle(x.device))
    if st != 0:
        raise GdnError(st, "gdn_rope3d")
    return out


class FrameStream:
    """Chunk-causal streaming through a device-side frame queue
    (gdn_frame_stream): one persistent launch serves frames as they are
    posted, keeping the state on chip, with no launch per frame.

    q, k, v, out: [ring, B, H, S, D] bf16 rings and gamma, beta: [ring, B, H]
    fp32 rings on the device; frame n lives in slot n % ring. Fill a slot
    (before the launch, or by copies from pinned host memory), then post();
    wait(n) returns once frames 0..n-1 are complete. close() stops the kernel
    and returns the final state. The counters live in pinned host memory.

    While the launch runs it holds its SMs and waits for the host, so between
    construction and close() the host may only post, wait, and copy between
    pinned host memory and pre-allocated device buffers on streams of its own.
    A kernel on the default stream, or an allocation, can be ordered after
    the running launch by CUDA's implicit synchronisation and then wait for it
    (the launch gives up after idle_timeout_s and reports a timeout).

    rope=(grid_w, t0) turns q and k by 3D RoPE inside the kernel, frame n of
    the queue as frame index t0 + n (gdn_frame_stream_rope).
    """

    STOP = -(1 << 63)    # bit 63 of the posted counter, as a signed int64

    def __init__(self, q, k, v, gamma, beta, out=None, state_in=None, *, want_state=True,
                 idle_timeout_s=10.0, delta=True, stream=None, rope=None):
        if q.dim() != 5 or q.dtype != torch.bfloat16 or q.device.type != "cuda":
            raise ValueError("q must be a [ring,B,H,S,D] bfloat16 CUDA tensor")
        R, B, H, S, D = q.shape
        dev = q.device
        for name, t in (("k", k), ("v", v)):
            _check(t, name, torch.bfloat16, q.shape, dev)
        _check(gamma, "gamma", torch.float32, (R, B, H), dev)
        _check(beta, "beta", torch.float32, (R, B, H), dev)
        if state_in is not None:
            _check(state_in, "state_in", torch.float32, (B, H, D, D), dev)
        self.out = torch.empty_like(q) if out is None else out
        _check(self.out, "out", torch.bfloat16, q.shape, dev)
        self.state = torch.empty((B, H, D, D), dtype=torch.float32, device=dev) if want_state else None
        # posted at word 0, done at word 16: different 128-byte lines, since the
        # host polls one while the device reads the other
        self.counters = torch.zeros(32, dtype=torch.int64, pin_memory=True)
        self._c = self.counters.numpy()     # the same pinned words, without torch's dispatch
        self.slots = torch.zeros(R + 2, dtype=torch.int32, device=dev)   # relay, then per slot
        self.stream = stream or torch.cuda.Stream(dev)
        self.stream.wait_stream(torch.cuda.current_stream(dev))   # the zeroed counters, the rings
        self.ring, self.posted = R, 0
        self._keep = (q, k, v, gamma, beta, state_in)
        base = self.counters.data_ptr()
        L = lib()
        common = (_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in),
                  _ptr(self.state), _ptr(self.out), B, H, S, D, R, ctypes.c_void_p(base),
                  ctypes.c_void_p(base + 128), _ptr(self.slots), int(idle_timeout_s * 1e9))
        flags = 0 if delta else FLAG_NO_DELTA
        with torch.cuda.device(dev):
            if rope is None:
                st = L.gdn_frame_stream(*common, flags, ctypes.c_void_p(self.stream.cuda_stream))
            else:
                st = L.gdn_frame_stream_rope(*common, int(rope[0]), int(rope[1]), flags,
                                             ctypes.c_void_p(self.stream.cuda_stream))
        if st != 0:
            raise GdnError(st, "gdn_frame_stream_rope" if rope is not None else "gdn_frame_stream")

    def post(self, frames=1):
        """Frames posted so far += frames (their slots must hold their inputs)."""
        self.posted += frames
        self._c[0] = self.posted

    def done(self) -> int:
        return int(self._c[16])

    def wait(self, n, timeout_s=10.0):
        """Polls until frames 0..n-1 are done; returns the time it waited."""
        import time
        c = self._c
        if c[16] >= n:
            return 0.0
        t0 = time.perf_counter()
        while c[16] < n:
            if time.perf_counter() - t0 > timeout_s:
                raise TimeoutError(f"frame stream: {int(c[16])} of {n} frames done")
        return time.perf_counter() - t0

    def close(self):
        """Stops the kernel after the posted frames; returns the final state."""
        self._c[0] = self.posted + self.STOP
        self.stream.synchronize()
        st = device_status()
        if st != 0:
            raise GdnError(st, "gdn_frame_stream")
        return self.state


def frame_scan_host(q, k, v, gamma, beta, state_in=None, *, device=None, stream=None,
                    staging=None, out_host=None, state_host=None, groups=8):
    """End-to-end call on HOST tensors: copies the inputs to the GPU, runs the
    scan there, copies out and the final state back, and waits for them.

    Heads are independent and contiguous in [B,H,T,S,D], so the work is cut
    into `groups` groups of heads and pipelined over three streams: the
    inputs of one group cross PCIe while the previous group is scanned and the
    one before it is copied back. Pass pinned tensors for asynchronous copies.
    `staging` may hold reusable device buffers (a dict filled on the first
    call) and out_host/state_host reusable pinned outputs. Returns
    (out_host, state_host) once everything is back."""
    device = torch.device(device or "cuda")
    stream = stream or torch.cuda.current_stream(device)
    staging = {} if staging is None else staging
    B, H, T, S, D = q.shape
    heads = B * H
    sshape = (B, H, D, D)
    if out_host is None:
        out_host = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if state_host is None:
        state_host = torch.empty(sshape, dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(device):
        def dev(name, shape, dtype):
            buf = staging.get(name)
            if buf is None or tuple(buf.shape) != tuple(shape) or buf.dtype != dtype:
                buf = torch.empty(shape, dtype=dtype, device=device)
                staging[name] = buf
            return buf
        flat = lambda t, *rest: t.reshape(heads, *rest)
        hq, hk, hv = (flat(x, 1, T, S, D) for x in (q, k, v))
        hg, hb = flat(gamma, 1, T), flat(beta, 1, T)
        hs = None if state_in is None else flat(state_in, 1, D, D)
        ho, hso = flat(out_host, 1, T, S, D), flat(state_host, 1, D, D)
        dq, dk, dv = (dev(n, (heads, 1, T, S, D), q.dtype) for n in ("q", "k", "v"))
        dg, db = dev("gamma", (heads, 1, T), torch.float32), dev("beta", (heads, 1, T), torch.float32)
        ds = None if state_in is None else dev("state_in", (heads, 1, D, D), torch.float32)
        do = dev("out", (heads, 1, T, S, D), q.dtype)
        dso = dev("state_out", (heads, 1, D, D), torch.float32)
        copy_in = staging.setdefault("copy_in", torch.cuda.Stream(device))
        copy_out = staging.setdefault("copy_out", torch.cuda.Stream(device))
        n = max(1, min(int(groups), heads))
        bounds = [heads * g // n for g in range(n + 1)]
        copy_in.wait_stream(stream)          # the buffers are free once earlier work is done
        copy_out.wait_stream(stream)
        for g in range(n):
            a, b = bounds[g], bounds[g + 1]
            if a == b:
                continue
            with torch.cuda.stream(copy_in):
                for dst, src in ((dq, hq), (dk, hk), (dv, hv), (dg, hg), (db, hb), (ds, hs)):
                    if src is not None:
                        dst[a:b].copy_(src[a:b], non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(copy_in)
            stream.wait_event(loaded)
            with torch.cuda.stream(stream):
                frame_scan(dq[a:b], dk[a:b], dv[a:b], dg[a:b], db[a:b],
                           None if ds is None else ds[a:b], out=do[a:b], state_out=dso[a:b])
                scanned = torch.cuda.Event()
                scanned.record(stream)
            copy_out.wait_event(scanned)
            with torch.cuda.stream(copy_out):
                ho[a:b].copy_(do[a:b], non_blocking=True)
                hso[a:b].copy_(dso[a:b], non_blocking=True)
        stream.wait_stream(copy_out)
        stream.synchronize()
    return out_host, state_host
