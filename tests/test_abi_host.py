"""Host-side checks of the C ABI (no GPU needed): the library builds and loads,
it exports every function the header declares, and argument checks return
their status before anything is enqueued (so fake device addresses are fine)."""
import ctypes
import os
import re

import pytest

import chunked_gated_delta_13_b200 as sf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sf_gdn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sf_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = sf.lib()
    names = declared_functions()
    assert names, "no declarations parsed"
    assert sorted(names) == sorted(sf.EXPORTED_SYMBOLS)
    for name in names:
        assert hasattr(L, name), name


def test_status_strings():
    L = sf.lib()
    for code, name in enumerate(sf.STATUS_NAMES):
        assert L.sf_status_str(code).decode() == name


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced: the checks return first


def fake(off=0):
    return ctypes.c_void_p(FAKE + off)


def call_fwd(shape, q=fake(), k=fake(), v=fake(), g=fake(), beta=fake(), S_in=None, o=fake(),
             S_out=None, ws=fake(), nbytes=1 << 40):
    return sf.lib().sf_gdn_fwd(ctypes.byref(shape), q, k, v, g, beta, S_in, o, S_out, ws, nbytes,
                               None)


def call_bwd(shape, **kw):
    args = dict(q=fake(), k=fake(), v=fake(), g=fake(), beta=fake(), S_in=None, dO=fake(),
                dS_out=None, dq=fake(), dk=fake(), dv=fake(), dg=fake(), dbeta=fake(),
                dS_in=None, ws=fake(), nbytes=1 << 40)
    args.update(kw)
    a = args
    return sf.lib().sf_gdn_bwd(ctypes.byref(shape), a["q"], a["k"], a["v"], a["g"], a["beta"],
                               a["S_in"], a["dO"], a["dS_out"], a["dq"], a["dk"], a["dv"], a["dg"],
                               a["dbeta"], a["dS_in"], a["ws"], a["nbytes"], None)


def test_invalid_shapes():
    bad = [sf.make_shape(-1, 1, 64, 64, 64), sf.make_shape(1, 1, -5, 64, 64)]
    for s in bad:
        assert call_fwd(s) == 1
    s = sf.make_shape(1, 1, 64, 64, 64)
    s.io = 7
    assert call_fwd(s) == 1
    s = sf.make_shape(1, 1, 64, 64, 64)
    s.use_beta = 3
    assert call_fwd(s) == 1
    s = sf.make_shape(1, 1, 64, 64, 64, scale=float("nan"))
    assert call_fwd(s) == 1
    assert sf.lib().sf_gdn_fwd(None, fake(), fake(), fake(), fake(), fake(), None, fake(), None,
                               fake(), 1, None) == 1


def test_unsupported_sizes():
    assert call_fwd(sf.make_shape(1, 1, 64, 96, 64)) == 2
    assert call_fwd(sf.make_shape(1, 1, 64, 64, 256)) == 2
    assert call_fwd(sf.make_shape(1, 1, 64, 64, 64, C=48)) == 2
    assert call_fwd(sf.make_shape(300, 300, 64, 64, 64)) == 2


def test_null_pointers_and_beta_flag():
    s = sf.make_shape(1, 2, 64, 64, 64)
    assert call_fwd(s, q=None) == 1
    assert call_fwd(s, o=None) == 1
    assert call_fwd(s, beta=None) == 1            # use_beta=1 needs beta
    s_off = sf.make_shape(1, 2, 64, 64, 64, use_beta=False)
    assert call_fwd(s_off) == 1                    # beta given although the beta path is off
    assert call_bwd(s, dq=None) == 1
    assert call_bwd(s, dbeta=None) == 1
    assert call_bwd(s_off, beta=None) == 1        # dbeta given without beta


def test_alignment():
    s = sf.make_shape(1, 2, 64, 64, 64)
    assert call_fwd(s, k=fake(8)) == 3
    assert call_fwd(s, S_in=fake(4)) == 3
    assert call_bwd(s, dg=fake(2)) == 3


def test_workspace_checks():
    s = sf.make_shape(1, 2, 200, 64, 64, C=64)
    need = sf.fwd_workspace_bytes(s)
    assert need > 0
    assert call_fwd(s, ws=None, nbytes=0) == 4
    assert call_fwd(s, nbytes=need - 1) == 4
    assert sf.bwd_workspace_bytes(s) >= need
    assert call_bwd(s, nbytes=sf.bwd_workspace_bytes(s) - 1) == 4
    assert sf.fwd_workspace_bytes(sf.make_shape(1, 2, 0, 64, 64)) == 0
    assert sf.fwd_workspace_bytes(sf.make_shape(1, 1, 64, 100, 64)) == 0


def test_segment_run_checks():
    s = sf.make_shape(1, 2, 256, 64, 64)
    L = sf.lib()
    nb = sf.segment_workspace_bytes(s, 4)
    assert nb > 0
    assert sf.segment_workspace_bytes(s, 0) == 0
    assert sf.segment_workspace_bytes(s, 2, [100, 100]) == 0      # lengths must sum to T
    assert sf.segment_workspace_bytes(s, 2, [0, 256]) > 0

    def run(N, seg, nbytes):
        arr = None if seg is None else (ctypes.c_int * N)(*seg)
        return L.sf_segment_run(ctypes.byref(s), N, arr, fake(), fake(), fake(), fake(), fake(),
                                None, None, None, fake(), None, None, None, None, None, None, None,
                                fake(), nbytes, None)
    assert run(0, None, nb) == 1
    assert run(2, [100, 100], nb) == 1
    assert run(4, None, nb - 1) == 4


def test_path_and_launch_counts():
    s = sf.make_shape(1, 2, 256, 64, 64, io="f32")
    assert sf.path(s) == "simt"
    assert sf.launches(s, False) >= 1 and sf.launches(s, True) >= 1
    assert sf.path(sf.make_shape(1, 1, 64, 100, 64)) is None


def test_cpu_tensors_rejected():
    torch = pytest.importorskip("torch")
    q = torch.zeros(1, 1, 8, 16)
    with pytest.raises(RuntimeError):
        sf.fwd(q, q, q, torch.zeros(1, 1, 8), torch.zeros(1, 1, 8))


def test_pipelined_segment_workspace_matches_the_documented_size():
    """Tensor-core segment chain: every piece keeps its forward and intra-chunk
    intermediates, 8 + 4 dk + 4 C + 6 dv + 4 dk dv / C bytes per token per head
    (2568 at dk = dv = 128, C = 64), plus three pieces' backward tiles and the
    fp32 boundary states; the pieces do not depend on how the caller splits T."""
    B, H, T, d, C = 1, 16, 65536, 128, 64
    s = sf.make_shape(B, H, T, d, d, C, "bf16")
    assert sf.path(s) == "tc"
    per_token = 8 + 4 * d + 4 * C + 6 * d + 4 * d * d // C
    assert per_token == 2568
    pieces = T // 4096
    keep = B * H * T * per_token
    slots = 3 * B * H * (4096 // C) * (2 * d * C + 2 * d * d)
    states = (pieces + 3) * B * H * d * d * 4
    expect = keep + slots + states
    for N in (1, 4, 16):
        got = sf.segment_workspace_bytes(s, N)
        assert expect <= got <= expect * 1.001, (N, got, expect)
    # a ragged split adds pieces, each with its own boundary state
    got = sf.segment_workspace_bytes(s, 3, [100, 65336, 100])
    assert got > expect


def test_timer_api_without_launches():
    """The native launch timer needs no GPU until a kernel runs: enabling with
    zero capacity, reading nothing and freeing are host-only."""
    L = sf.lib()
    L.sf_timer_free()
    assert L.sf_timer_count() == 0
    assert L.sf_timer_enable(-1) == 1          # SF_ERR_INVALID_ARG
    assert L.sf_timer_enable(0) == 0
    assert L.sf_timer_count() == 0
    name, ms = ctypes.c_char_p(), ctypes.c_float()
    assert L.sf_timer_read(0, ctypes.byref(name), ctypes.byref(ms)) == 1
    L.sf_timer_disable()
    L.sf_timer_free()


def test_bounded_memory_workspace():
    """The bounded-memory chain needs the boundary states plus one segment's
    backward workspace: far less than the pipelined chain on the tensor-core
    path, the same on the CUDA-core path (which always runs sequentially)."""
    tc = sf.make_shape(1, 16, 65536, 128, 128, 64, "bf16")
    full = sf.segment_workspace_bytes(tc, 16)
    small = sf.segment_workspace_bytes(tc, 16, bounded_memory=True)
    one = sf.bwd_workspace_bytes(sf.make_shape(1, 16, 4096, 128, 128, 64, "bf16"))
    state = 16 * 128 * 128 * 4
    assert small == 19 * state + one + 256
    assert small * 10 < full
    simt = sf.make_shape(1, 2, 256, 64, 64, 64, "f32")
    assert sf.segment_workspace_bytes(simt, 2) == sf.segment_workspace_bytes(simt, 2, bounded_memory=True)
    assert sf.lib().sf_segment_min_workspace_bytes(ctypes.byref(tc), 0, None) == 0
