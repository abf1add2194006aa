"""fp64 CPU oracle for the gated delta-rule layer with an explicit boundary state.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library in ``chunked_gated_delta_13_b200`` and never imports it.

The arithmetic lives in ``gdn_oracle.c`` (token-by-token recurrence and its
reverse-time adjoint; StateFlow, arXiv 2608.06838, section 2.1).  This module
compiles it with gcc on first use, and wraps it for numpy fp64 arrays.

``segment_run`` is the plain definition of the sequence split and the two
boundary-state chains (StateFlow section 3.1: the split X = C_0 || ... ||
C_{N-1}, the chunk forward Fwd(C_in, S_in) -> (C_out, S_out) and backward
Bwd(C_in, S_in, dC_out, dS_out) -> (dC_in, dS_in), with the state handed
forward S_{i+1}^in = S_i^out and the state gradient handed backward
dS_i^out = dS_{i+1}^in, the last two as restated by the page's review).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (plain fp64 C + OpenMP) into ``oracle/liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.POINTER(ctypes.c_double)
            i = ctypes.c_int
            lib.oracle_gdn_fwd.argtypes = [i, i, i, i, i, P, P, P, P, P, P, ctypes.c_double, P, P]
            lib.oracle_gdn_fwd.restype = i
            lib.oracle_gdn_bwd.argtypes = [i, i, i, i, i, P, P, P, P, P, P, ctypes.c_double,
                                           P, P, P, P, P, P, P, P, i]
            lib.oracle_gdn_bwd.restype = i
            lib.oracle_threads.argtypes = []
            lib.oracle_threads.restype = i
            _lib = lib
    return _lib


def threads() -> int:
    """OpenMP threads the oracle uses (one head per thread at a time)."""
    return int(_load().oracle_threads())


def _c(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, v):
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    return B, H, T, dk, dv


def gdn_fwd(q, k, v, g, beta, S_in=None, scale=1.0):
    """Forward of one segment.

    q, k: [B,H,T,dk]; v: [B,H,T,dv]; g, beta: [B,H,T] (beta=None: beta path off);
    S_in: [B,H,dk,dv] or None (zeros).  Returns (o [B,H,T,dv], S_out [B,H,dk,dv]).
    """
    q, k, v, g = _c(q), _c(k), _c(v), _c(g)
    beta = None if beta is None else _c(beta)
    S_in = None if S_in is None else _c(S_in)
    B, H, T, dk, dv = _dims(q, v)
    o = np.zeros((B, H, T, dv))
    S_out = np.zeros((B, H, dk, dv))
    rc = _load().oracle_gdn_fwd(B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                _ptr(S_in), float(scale), _ptr(o), _ptr(S_out))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn_fwd failed ({rc})")
    return o, S_out


def gdn_bwd(q, k, v, g, beta, S_in, dO, dS_out=None, scale=1.0, ckpt=64):
    """Backward of one segment by the reverse-time adjoint.

    Returns a dict with dq, dk, dv, dg, dbeta (None when beta is None) and dS_in.
    """
    q, k, v, g, dO = _c(q), _c(k), _c(v), _c(g), _c(dO)
    beta = None if beta is None else _c(beta)
    S_in = None if S_in is None else _c(S_in)
    dS_out = None if dS_out is None else _c(dS_out)
    B, H, T, dk, dv = _dims(q, v)
    dq = np.zeros((B, H, T, dk))
    dkk = np.zeros((B, H, T, dk))
    dvv = np.zeros((B, H, T, dv))
    dg = np.zeros((B, H, T))
    dbeta = np.zeros((B, H, T)) if beta is not None else None
    dS_in = np.zeros((B, H, dk, dv))
    rc = _load().oracle_gdn_bwd(B, H, T, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                _ptr(S_in), float(scale), _ptr(dO), _ptr(dS_out), _ptr(dq),
                                _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(dbeta), _ptr(dS_in), int(ckpt))
    if rc != 0:
        raise RuntimeError(f"oracle_gdn_bwd failed ({rc})")
    return {"dq": dq, "dk": dkk, "dv": dvv, "dg": dg, "dbeta": dbeta, "dS_in": dS_in}


def loss(o, S_out, dO, dS_out):
    """The scalar whose gradients gdn_bwd returns: sum <o,dO> + <S_out,dS_out>."""
    val = float(np.sum(np.asarray(o, np.float64) * np.asarray(dO, np.float64)))
    if dS_out is not None:
        val += float(np.sum(np.asarray(S_out, np.float64) * np.asarray(dS_out, np.float64)))
    return val


def segment_bounds(T, N=None, seg_len=None):
    """Start/stop of each segment of the split X = C_0 || ... || C_{N-1}."""
    if seg_len is None:
        if N is None or N <= 0:
            raise ValueError("need N or seg_len")
        base, rem = divmod(T, N)
        seg_len = [base + (1 if i < rem else 0) for i in range(N)]
    if sum(seg_len) != T or any(s < 0 for s in seg_len):
        raise ValueError("segment lengths must be non-negative and sum to T")
    out, t = [], 0
    for s in seg_len:
        out.append((t, t + s))
        t += s
    return out


def segment_run(q, k, v, g, beta, S_in, dO, dS_out, N=None, seg_len=None, scale=1.0):
    """Split one sequence into segments and run them in order with state handoff.

    Forward over segments i = 0..N-1 with S_{i+1}^in = S_i^out, then backward over
    i = N-1..0 with dS_i^out = dS_{i+1}^in.  Returns (o, S_out, grads dict).
    """
    q, k, v, g, dO = _c(q), _c(k), _c(v), _c(g), _c(dO)
    beta = None if beta is None else _c(beta)
    B, H, T, dk, dv = _dims(q, v)
    bounds = segment_bounds(T, N, seg_len)
    S = [np.zeros((B, H, dk, dv)) if S_in is None else _c(S_in)]
    o = np.zeros((B, H, T, dv))
    for (a, b) in bounds:
        o_i, S_next = gdn_fwd(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], g[:, :, a:b],
                              None if beta is None else beta[:, :, a:b], S[-1], scale)
        o[:, :, a:b] = o_i
        S.append(S_next)
    grads = {"dq": np.zeros((B, H, T, dk)), "dk": np.zeros((B, H, T, dk)),
             "dv": np.zeros((B, H, T, dv)), "dg": np.zeros((B, H, T)),
             "dbeta": None if beta is None else np.zeros((B, H, T))}
    dS = np.zeros((B, H, dk, dv)) if dS_out is None else _c(dS_out)
    for i in range(len(bounds) - 1, -1, -1):
        a, b = bounds[i]
        gr = gdn_bwd(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], g[:, :, a:b],
                     None if beta is None else beta[:, :, a:b], S[i], dO[:, :, a:b], dS, scale)
        for name in ("dq", "dk", "dv", "dg"):
            grads[name][:, :, a:b] = gr[name]
        if beta is not None:
            grads["dbeta"][:, :, a:b] = gr["dbeta"]
        dS = gr["dS_in"]
    grads["dS_in"] = dS
    return o, S[-1], grads
