"""The forward entry point that allocates nothing (sf_gdn_fwd_noalloc).

It serves callers that cannot hand the library a workspace, such as an engine
whose device memory is planned up front or code that must not call cudaMalloc
on its hot path.  It takes its scratch from a fixed array the library keeps on
each GPU.  This file is named so pytest collects it last; it passes in a fresh
process as well as after the rest of the suite.
"""
import ctypes

import pytest
import torch

import chunked_gated_delta_13_b200 as sf
from chunked_gated_delta_13_b200.inputs import Workload, make_inputs
from gpu_util import to_device

pytestmark = pytest.mark.gpu

SCRATCH = 32 << 20  # SF_NOALLOC_SCRATCH_BYTES


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_fwd(d, C, scale=1.0):
    q, v = d["q"], d["v"]
    B, H, T, dk = q.shape
    shape = sf.make_shape(B, H, T, dk, v.shape[-1], C, "bf16" if q.dtype == torch.bfloat16 else "f32",
                          d["beta"] is not None, scale)
    o = torch.full_like(v, float("nan"))
    S_out = torch.full((B, H, dk, v.shape[-1]), float("nan"), device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sf.lib().sf_gdn_fwd_noalloc(ctypes.byref(shape), _ptr(q), _ptr(d["k"]), _ptr(v), _ptr(d["g"]),
                                     _ptr(d["beta"]), _ptr(d["S_in"]), _ptr(o), _ptr(S_out), stream)
    return rc, o, S_out


@pytest.mark.parametrize("w", [
    Workload("na_bf16", B=1, H=4, T=3 * 64 + 29, dk=128, dv=128, C=64, io="bf16", S_in_std=0.05,
             g_shift=-3.0),
    Workload("na_f32", B=2, H=2, T=150, dk=64, dv=32, C=32, io="f32", S_in_std=0.05),
])
def test_noalloc_forward_matches_workspace_forward(w):
    """The scratch-backed forward runs the same kernels as sf_gdn_fwd, so its
    outputs must be bit-equal.  Before each compared call the scratch is filled
    by a call on other inputs (another seed, a longer sequence that still fits),
    so reading anything stale would show."""
    d = to_device(make_inputs(w))
    o_ref, S_ref = sf.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], C=w.C)
    torch.cuda.synchronize()
    T_dirty = 4000 if w.io == "bf16" else 2000
    dirty = to_device(make_inputs(w.with_(T=T_dirty, seed=w.seed + 1, g_shift=-4.0)))
    for _ in range(2):  # two calls in a row: the shared scratch keeps the previous call's contents
        rc, _, _ = _noalloc_fwd(dirty, w.C)
        assert rc == 0, sf.STATUS_NAMES[rc]
        rc, o, S_out = _noalloc_fwd(d, w.C)
        torch.cuda.synchronize()
        assert rc == 0, sf.STATUS_NAMES[rc]
        assert torch.equal(o, o_ref)
        assert torch.equal(S_out, S_ref)


def test_noalloc_rejects_shapes_beyond_the_scratch():
    big = sf.make_shape(1, 16, 65536, 128, 128, 64, "bf16", True, 1.0)
    assert sf.fwd_workspace_bytes(big) > SCRATCH
    fake = ctypes.c_void_p(0x7F0000000000)
    rc = sf.lib().sf_gdn_fwd_noalloc(ctypes.byref(big), fake, fake, fake, fake, fake, None, fake, None,
                                     None)
    assert rc == 4  # SF_ERR_WORKSPACE, nothing enqueued
