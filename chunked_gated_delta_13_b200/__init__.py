"""Chunked gated delta-rule (Gated DeltaNet) forward/backward with an explicit
boundary state, for NVIDIA B200 (sm_100a).

This module is the Python binding of ``libsf_gdn.so``: argument marshalling
only.  PyTorch provides device memory and the stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: a
missing library or a CPU tensor raises.

Entry points mirror the C ABI in ``include/sf_gdn.h``:
  fwd(q, k, v, g, beta, S_in)                       -> (o, S_out)
  bwd(q, k, v, g, beta, S_in, dO, dS_out)           -> dict of gradients
  segment_run(..., N or seg_len)                    -> (o, S_out, gradients)
  conv_fwd / conv_bwd / conv_segment_run            the short causal convolution
                                                    with its boundary state
  kda_fwd / kda_bwd                                 the delta rule with a per-channel
                                                    (diagonal) decay
The operations are StateFlow's chunk Fwd/Bwd and its sequence split with the
state handed forward and the state gradient handed backward (arXiv 2608.06838,
sections 2.1 and 3.1).
"""
from __future__ import annotations

import ctypes
import os
import threading

from ._build import LIB, build, needs_build

__all__ = ["Shape", "ConvShape", "KdaShape", "kda_fwd", "kda_bwd", "make_conv_shape", "conv_fwd", "conv_bwd", "conv_segment_run", "SFError", "lib", "fwd", "bwd", "segment_run", "make_shape", "path", "device_check",
           "launches", "set_launch_hook", "timer_enable", "timer_disable", "timer_count", "timer_results", "timer_timeline", "timer_free",
           "fwd_workspace_bytes", "bwd_workspace_bytes", "segment_workspace_bytes",
           "EXPORTED_SYMBOLS"]

SF_F32, SF_BF16 = 0, 1

STATUS_NAMES = ["SF_OK", "SF_ERR_INVALID_ARG", "SF_ERR_UNSUPPORTED", "SF_ERR_ALIGNMENT",
                "SF_ERR_WORKSPACE", "SF_ERR_CUDA", "SF_ERR_TIMEOUT"]

EXPORTED_SYMBOLS = [
    "sf_status_str", "sf_last_cuda_error", "sf_gdn_fwd_workspace_bytes",
    "sf_gdn_bwd_workspace_bytes", "sf_gdn_fwd", "sf_gdn_bwd", "sf_segment_workspace_bytes",
    "sf_segment_run", "sf_segment_min_workspace_bytes", "sf_gdn_path", "sf_gdn_launches", "sf_set_launch_hook", "sf_gdn_fwd_noalloc",
    "sf_device_check", "sf_timer_enable", "sf_timer_disable", "sf_timer_count", "sf_timer_read",
    "sf_timer_free", "sf_timer_read_at", "sf_conv_workspace_bytes", "sf_conv_fwd", "sf_conv_bwd",
    "sf_conv_segment_workspace_bytes", "sf_conv_segment_run", "sf_kda_workspace_bytes", "sf_kda_fwd",
    "sf_kda_bwd",
]

HOOK_T = ctypes.CFUNCTYPE(None, ctypes.c_char_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p)


class Shape(ctypes.Structure):
    """Mirror of ``sf_gdn_shape``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("C", ctypes.c_int),
                ("io", ctypes.c_int), ("use_beta", ctypes.c_int), ("scale", ctypes.c_float)]


class ConvShape(ctypes.Structure):
    """Mirror of ``sf_conv_shape``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("d", ctypes.c_int),
                ("K", ctypes.c_int), ("io", ctypes.c_int), ("act", ctypes.c_int)]


class KdaShape(ctypes.Structure):
    """Mirror of ``sf_kda_shape``."""
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("io", ctypes.c_int), ("use_beta", ctypes.c_int), ("scale", ctypes.c_float)]


class SFError(RuntimeError):
    """A non-zero sf_status returned by the library."""

    def __init__(self, status: int, msg: str = ""):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else f"status {status}"
        super().__init__(f"{name}{': ' + msg if msg else ''}")


_lock = threading.Lock()
_lib = None


def lib():
    """Load libsf_gdn.so, building it in-tree first if it is missing or older than
    any of its sources (a failed build raises).  The environment variable
    SF_GDN_LIB may name a prebuilt library to load as it is instead."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = os.environ.get("SF_GDN_LIB")
        if path:
            # explicit opt-in to a prebuilt library (no rebuild, no staleness check)
            if not os.path.exists(path):
                raise RuntimeError(f"SF_GDN_LIB names a missing file: {path}")
        else:
            path = LIB
            if needs_build():
                # a library older than its sources is never loaded: a failed
                # rebuild (no nvcc, a compile error) raises instead
                try:
                    build()
                except Exception as exc:
                    raise RuntimeError(f"libsf_gdn.so is missing or older than its sources and could "
                                       f"not be rebuilt: {exc}") from exc
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        SP = ctypes.POINTER(Shape)
        L.sf_status_str.argtypes = [ctypes.c_int]
        L.sf_status_str.restype = ctypes.c_char_p
        L.sf_last_cuda_error.argtypes = []
        L.sf_last_cuda_error.restype = ctypes.c_char_p
        for name in ("sf_gdn_fwd_workspace_bytes", "sf_gdn_bwd_workspace_bytes"):
            getattr(L, name).argtypes = [SP]
            getattr(L, name).restype = ctypes.c_size_t
        for name in ("sf_segment_workspace_bytes", "sf_segment_min_workspace_bytes"):
            getattr(L, name).argtypes = [SP, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
            getattr(L, name).restype = ctypes.c_size_t
        L.sf_gdn_fwd.argtypes = [SP] + [P] * 8 + [P, ctypes.c_size_t, P]
        L.sf_gdn_fwd.restype = ctypes.c_int
        L.sf_gdn_bwd.argtypes = [SP] + [P] * 14 + [P, ctypes.c_size_t, P]
        L.sf_gdn_bwd.restype = ctypes.c_int
        L.sf_segment_run.argtypes = ([SP, ctypes.c_int, ctypes.POINTER(ctypes.c_int)] + [P] * 16
                                     + [P, ctypes.c_size_t, P])
        L.sf_segment_run.restype = ctypes.c_int
        L.sf_gdn_path.argtypes = [SP]
        L.sf_gdn_path.restype = ctypes.c_char_p
        L.sf_gdn_launches.argtypes = [SP, ctypes.c_int]
        L.sf_gdn_launches.restype = ctypes.c_int
        L.sf_device_check.argtypes = []
        L.sf_device_check.restype = ctypes.c_int
        L.sf_gdn_fwd_noalloc.argtypes = [SP] + [P] * 8 + [P]
        L.sf_gdn_fwd_noalloc.restype = ctypes.c_int
        L.sf_set_launch_hook.argtypes = [HOOK_T, ctypes.c_void_p]
        L.sf_set_launch_hook.restype = None
        L.sf_timer_enable.argtypes = [ctypes.c_int]
        L.sf_timer_enable.restype = ctypes.c_int
        L.sf_timer_disable.argtypes = []
        L.sf_timer_disable.restype = None
        L.sf_timer_count.argtypes = []
        L.sf_timer_count.restype = ctypes.c_int
        L.sf_timer_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float)]
        L.sf_timer_read.restype = ctypes.c_int
        L.sf_timer_read_at.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                                       ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
        L.sf_timer_read_at.restype = ctypes.c_int
        L.sf_timer_free.argtypes = []
        L.sf_timer_free.restype = None
        CP = ctypes.POINTER(ConvShape)
        L.sf_conv_workspace_bytes.argtypes = [CP]
        L.sf_conv_workspace_bytes.restype = ctypes.c_size_t
        L.sf_conv_fwd.argtypes = [CP] + [P] * 5 + [P]
        L.sf_conv_fwd.restype = ctypes.c_int
        L.sf_conv_bwd.argtypes = [CP] + [P] * 9 + [P, ctypes.c_size_t, P]
        L.sf_conv_bwd.restype = ctypes.c_int
        L.sf_conv_segment_workspace_bytes.argtypes = [CP, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        L.sf_conv_segment_workspace_bytes.restype = ctypes.c_size_t
        L.sf_conv_segment_run.argtypes = ([CP, ctypes.c_int, ctypes.POINTER(ctypes.c_int)] + [P] * 10
                                          + [P, ctypes.c_size_t, P])
        L.sf_conv_segment_run.restype = ctypes.c_int
        KP = ctypes.POINTER(KdaShape)
        L.sf_kda_workspace_bytes.argtypes = [KP, ctypes.c_int]
        L.sf_kda_workspace_bytes.restype = ctypes.c_size_t
        L.sf_kda_fwd.argtypes = [KP] + [P] * 8 + [P]
        L.sf_kda_fwd.restype = ctypes.c_int
        L.sf_kda_bwd.argtypes = [KP] + [P] * 14 + [P, ctypes.c_size_t, P]
        L.sf_kda_bwd.restype = ctypes.c_int
        _lib = L
        return _lib


def _check(status: int):
    if status != 0:
        raise SFError(status, lib().sf_last_cuda_error().decode() if status == 5 else "")


def device_check():
    """Synchronise and raise SFError(SF_ERR_TIMEOUT) if a kernel gave up one of its
    bounded waits since the last check."""
    _check(lib().sf_device_check())


def make_shape(B, H, T, dk, dv, C=64, io="bf16", use_beta=True, scale=1.0) -> Shape:
    io_code = {"bf16": SF_BF16, "f32": SF_F32}[io]
    return Shape(int(B), int(H), int(T), int(dk), int(dv), int(C), io_code, int(bool(use_beta)),
                 float(scale))


def fwd_workspace_bytes(shape: Shape) -> int:
    return int(lib().sf_gdn_fwd_workspace_bytes(ctypes.byref(shape)))


def bwd_workspace_bytes(shape: Shape) -> int:
    return int(lib().sf_gdn_bwd_workspace_bytes(ctypes.byref(shape)))


def _seg_array(N, seg_len):
    if seg_len is None:
        return None
    if len(seg_len) != N:
        raise ValueError("seg_len must have N entries")
    return (ctypes.c_int * N)(*[int(x) for x in seg_len])


def segment_workspace_bytes(shape: Shape, N: int, seg_len=None, bounded_memory=False) -> int:
    """Workspace of segment_run: the fastest mode, or with bounded_memory the
    mode that keeps only the boundary states and recomputes each segment."""
    f = lib().sf_segment_min_workspace_bytes if bounded_memory else lib().sf_segment_workspace_bytes
    return int(f(ctypes.byref(shape), int(N), _seg_array(N, seg_len)))


def path(shape: Shape):
    p = lib().sf_gdn_path(ctypes.byref(shape))
    return None if p is None else p.decode()


def launches(shape: Shape, backward: bool) -> int:
    return int(lib().sf_gdn_launches(ctypes.byref(shape), int(bool(backward))))


_hook_ref = None


def set_launch_hook(fn):
    """Observe kernel launches: fn(kernel_name: str, after: bool, stream_handle: int)
    is called around every launch on the calling thread; None removes it."""
    global _hook_ref
    if fn is None:
        _hook_ref = None
        lib().sf_set_launch_hook(HOOK_T(), None)
        return

    def _cb(name, after, stream, user):
        fn(name.decode(), bool(after), stream or 0)

    _hook_ref = HOOK_T(_cb)
    lib().sf_set_launch_hook(_hook_ref, None)


def timer_enable(capacity: int):
    """Time the next `capacity` kernel launches with CUDA events recorded by the
    library itself on each launch's stream (see sf_timer_enable)."""
    _check(lib().sf_timer_enable(int(capacity)))


def timer_disable():
    lib().sf_timer_disable()


def timer_count() -> int:
    return int(lib().sf_timer_count())


def timer_results():
    """[(kernel_name, ms)] of the recorded launches, in launch order (waits for them)."""
    out = []
    name = ctypes.c_char_p()
    ms = ctypes.c_float()
    for i in range(lib().sf_timer_count()):
        _check(lib().sf_timer_read(i, ctypes.byref(name), ctypes.byref(ms)))
        out.append((name.value.decode(), float(ms.value)))
    return out


def timer_timeline():
    """[(kernel_name, start_ms, ms)] of the recorded launches, starts relative to
    the first launch's start (waits for them)."""
    out = []
    name = ctypes.c_char_p()
    t0 = ctypes.c_float()
    ms = ctypes.c_float()
    for i in range(lib().sf_timer_count()):
        _check(lib().sf_timer_read_at(i, ctypes.byref(name), ctypes.byref(t0), ctypes.byref(ms)))
        out.append((name.value.decode(), float(t0.value), float(ms.value)))
    return out


def timer_free():
    lib().sf_timer_free()


# ------------------------------------------------------------ torch glue ----

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io_of(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return "bf16"
    if t.dtype == torch.float32:
        return "f32"
    raise TypeError(f"q/k/v must be bf16 or fp32, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise RuntimeError("libsf_gdn runs on CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace too small: need {nbytes} bytes")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _shape_of(q, v, beta, C, scale):
    B, H, T, dk = q.shape
    return make_shape(B, H, T, dk, v.shape[-1], C, _io_of(q), beta is not None, scale)


def fwd(q, k, v, g, beta=None, S_in=None, *, C=64, scale=1.0, o=None, S_out=None,
        workspace=None, stream=None):
    """Forward of one segment.  Returns (o, S_out)."""
    torch = _torch()
    _need_cuda(q, k, v, g, beta, S_in)
    shape = _shape_of(q, v, beta, C, scale)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device)
    if S_out is None:
        S_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    ws = _workspace(fwd_workspace_bytes(shape), q.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().sf_gdn_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                            _ptr(S_in), _ptr(o), _ptr(S_out), _ptr(ws), nbytes, _stream(stream)))
    return o, S_out


def bwd(q, k, v, g, beta, S_in, dO, dS_out=None, *, C=64, scale=1.0, out=None, workspace=None,
        stream=None):
    """Backward of one segment.  Returns a dict: dq, dk, dv, dg, dbeta (None when
    the beta path is off) and dS_in."""
    torch = _torch()
    _need_cuda(q, k, v, g, beta, S_in, dO, dS_out)
    shape = _shape_of(q, v, beta, C, scale)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = {
            "dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
            "dg": torch.empty(B, H, T, dtype=torch.float32, device=q.device),
            "dbeta": None if beta is None else torch.empty(B, H, T, dtype=torch.float32,
                                                           device=q.device),
            "dS_in": torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device),
        }
    ws = _workspace(bwd_workspace_bytes(shape), q.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().sf_gdn_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                            _ptr(S_in), _ptr(dO), _ptr(dS_out), _ptr(out["dq"]), _ptr(out["dk"]),
                            _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbeta"]),
                            _ptr(out["dS_in"]), _ptr(ws), nbytes, _stream(stream)))
    return out


def segment_run(q, k, v, g, beta, S_in, dO, dS_out=None, *, N=1, seg_len=None, C=64, scale=1.0,
                out=None, workspace=None, stream=None, bounded_memory=False):
    """Run the sequence as N segments in order with state handoff (forward), then
    in reverse with state-gradient handoff (backward, skipped when dO is None).
    bounded_memory=True allocates only the bounded-memory workspace (boundary
    states plus one segment); a caller workspace picks the mode by its size.

    Returns (o, S_out, grads) where grads is None when dO is None."""
    torch = _torch()
    _need_cuda(q, k, v, g, beta, S_in, dO, dS_out)
    shape = _shape_of(q, v, beta, C, scale)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    if out is None:
        out = {"o": torch.empty(B, H, T, dv, dtype=q.dtype, device=q.device),
               "S_out": torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)}
        if dO is not None:
            out.update({
                "dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
                "dg": torch.empty(B, H, T, dtype=torch.float32, device=q.device),
                "dbeta": None if beta is None else torch.empty(B, H, T, dtype=torch.float32,
                                                               device=q.device),
                "dS_in": torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)})
    segs = _seg_array(N, seg_len)
    ws = _workspace(segment_workspace_bytes(shape, N, seg_len, bounded_memory), q.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    g_ = lambda name: _ptr(out.get(name)) if dO is not None else None
    _check(lib().sf_segment_run(ctypes.byref(shape), int(N), segs, _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(beta), _ptr(S_in), _ptr(dO), _ptr(dS_out),
                                _ptr(out["o"]), _ptr(out["S_out"]), g_("dq"), g_("dk"), g_("dv"),
                                g_("dg"), g_("dbeta"), g_("dS_in"), _ptr(ws), nbytes,
                                _stream(stream)))
    grads = None
    if dO is not None:
        grads = {n: out[n] for n in ("dq", "dk", "dv", "dg", "dbeta", "dS_in")}
    return out["o"], out["S_out"], grads


# ------------------------------------------------- short convolution glue ---

def make_conv_shape(B, H, T, d, K, io="bf16", act="silu") -> ConvShape:
    io_code = {"bf16": SF_BF16, "f32": SF_F32}[io]
    return ConvShape(int(B), int(H), int(T), int(d), int(K), io_code, {"none": 0, "silu": 1}[act])


def _conv_shape_of(x, w, act):
    B, H, T, d = x.shape
    return make_conv_shape(B, H, T, d, w.shape[-1], _io_of(x), act)


def conv_fwd(x, w, conv_in=None, *, act="silu", y=None, conv_out=None, stream=None):
    """Short causal convolution of one segment with its boundary state.
    x: [B,H,T,d] (bf16 or fp32); w: [H,d,K] fp32; conv_in: [B,H,K-1,d] (x's dtype)
    or None.  Returns (y, conv_out)."""
    torch = _torch()
    _need_cuda(x, w, conv_in)
    shape = _conv_shape_of(x, w, act)
    B, H, T, d = x.shape
    K = w.shape[-1]
    if y is None:
        y = torch.empty_like(x)
    if conv_out is None:
        conv_out = torch.empty(B, H, K - 1, d, dtype=x.dtype, device=x.device)
    _check(lib().sf_conv_fwd(ctypes.byref(shape), _ptr(x), _ptr(w), _ptr(conv_in), _ptr(y),
                             _ptr(conv_out), _stream(stream)))
    return y, conv_out


def conv_bwd(x, w, conv_in, dy, dconv_out=None, *, act="silu", dw_in=None, out=None, workspace=None,
             stream=None):
    """Backward of one segment.  Returns a dict: dx, dw (= dw_in + this segment's
    weight gradient) and dconv_in."""
    torch = _torch()
    _need_cuda(x, w, conv_in, dy, dconv_out, dw_in)
    shape = _conv_shape_of(x, w, act)
    B, H, T, d = x.shape
    K = w.shape[-1]
    if out is None:
        out = {"dx": torch.empty_like(x), "dw": torch.empty_like(w),
               "dconv_in": torch.empty(B, H, K - 1, d, dtype=torch.float32, device=x.device)}
    ws = _workspace(int(lib().sf_conv_workspace_bytes(ctypes.byref(shape))), x.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().sf_conv_bwd(ctypes.byref(shape), _ptr(x), _ptr(w), _ptr(conv_in), _ptr(dy),
                             _ptr(dconv_out), _ptr(out["dx"]), _ptr(dw_in), _ptr(out["dw"]),
                             _ptr(out["dconv_in"]), _ptr(ws), nbytes, _stream(stream)))
    return out


def conv_segment_run(x, w, conv_in, dy, dconv_out=None, *, N=1, seg_len=None, act="silu",
                     workspace=None, stream=None):
    """The convolution's segment chain: N segments forward with the state handed
    on, then (dy given) backward in reverse with its gradient handed back.
    Returns (y, conv_out, grads) with grads None when dy is None."""
    torch = _torch()
    _need_cuda(x, w, conv_in, dy, dconv_out)
    shape = _conv_shape_of(x, w, act)
    B, H, T, d = x.shape
    K = w.shape[-1]
    segs = _seg_array(N, seg_len)
    y = torch.empty_like(x)
    conv_out = torch.empty(B, H, K - 1, d, dtype=x.dtype, device=x.device)
    grads = None
    if dy is not None:
        grads = {"dx": torch.empty_like(x), "dw": torch.empty_like(w),
                 "dconv_in": torch.empty(B, H, K - 1, d, dtype=torch.float32, device=x.device)}
    need = int(lib().sf_conv_segment_workspace_bytes(ctypes.byref(shape), int(N), segs))
    if need == 0:
        raise SFError(1, "invalid convolution shape or segment lengths")
    ws = _workspace(need, x.device, workspace)
    g_ = (lambda n: _ptr(grads[n])) if grads is not None else (lambda n: None)
    _check(lib().sf_conv_segment_run(ctypes.byref(shape), int(N), segs, _ptr(x), _ptr(w),
                                     _ptr(conv_in), _ptr(dy), _ptr(dconv_out), _ptr(y),
                                     _ptr(conv_out), g_("dx"), g_("dw"), g_("dconv_in"), _ptr(ws),
                                     ws.numel(), _stream(stream)))
    return y, conv_out, grads


# ------------------------------------------------ per-channel decay glue ---

def _kda_shape_of(q, v, beta, scale):
    B, H, T, dk = q.shape
    return KdaShape(B, H, T, dk, v.shape[-1], SF_BF16 if _io_of(q) == "bf16" else SF_F32,
                    int(beta is not None), float(scale))


def kda_fwd(q, k, v, g, beta=None, S_in=None, *, scale=1.0, stream=None):
    """Forward of the delta rule with a per-channel decay; g: [B,H,T,dk] fp32.
    Returns (o, S_out)."""
    torch = _torch()
    _need_cuda(q, k, v, g, beta, S_in)
    shape = _kda_shape_of(q, v, beta, scale)
    B, H, T, dk = q.shape
    o = torch.empty(B, H, T, v.shape[-1], dtype=q.dtype, device=q.device)
    S_out = torch.empty(B, H, dk, v.shape[-1], dtype=torch.float32, device=q.device)
    _check(lib().sf_kda_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                            _ptr(o), _ptr(S_out), _stream(stream)))
    return o, S_out


def kda_bwd(q, k, v, g, beta, S_in, dO, dS_out=None, *, scale=1.0, workspace=None, stream=None):
    """Backward: dict dq, dk, dv, dg ([B,H,T,dk] fp32), dbeta, dS_in."""
    torch = _torch()
    _need_cuda(q, k, v, g, beta, S_in, dO, dS_out)
    shape = _kda_shape_of(q, v, beta, scale)
    B, H, T, dk = q.shape
    out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dg": torch.empty_like(g), "dbeta": None if beta is None else torch.empty_like(beta),
           "dS_in": torch.empty(B, H, dk, v.shape[-1], dtype=torch.float32, device=q.device)}
    ws = _workspace(int(lib().sf_kda_workspace_bytes(ctypes.byref(shape), 1)), q.device, workspace)
    nbytes = 0 if ws is None else ws.numel()
    _check(lib().sf_kda_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S_in),
                            _ptr(dO), _ptr(dS_out), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                            _ptr(out["dg"]), _ptr(out["dbeta"]), _ptr(out["dS_in"]), _ptr(ws), nbytes,
                            _stream(stream)))
    return out
