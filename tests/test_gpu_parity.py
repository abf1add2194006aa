"""Parity of the CUDA path (called through the C ABI) with the fp64 oracle.

Bars: max-relative error (max|gpu - oracle| / max|oracle|, per output tensor)
<= 1e-4 with fp32 I/O and <= 2e-2 with bf16 I/O and fp32 state; an N-segment
run is bit-identical to the 1-segment run when every segment length is a
multiple of the chunk length.
"""
import numpy as np
import pytest
import torch

import chunked_gated_delta_13_b200 as sf
from chunked_gated_delta_13_b200.inputs import CONFIGS, Workload, make_inputs
from gpu_util import compare, gpu_fwd_bwd, gpu_segments, oracle_fwd_bwd, to_device

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def small(**kw) -> Workload:
    base = dict(name="small", B=2, H=3, T=3 * 64 + 17, dk=64, dv=64, C=64, io="f32",
                S_in_std=0.05, dS_out_std=0.1)
    base.update(kw)
    return Workload(**base)


def check(w: Workload, tol, heads=None):
    inp = make_inputs(w)
    gpu = gpu_fwd_bwd(to_device(inp), w.C, w.scale)
    ref = oracle_fwd_bwd(inp, heads=heads, scale=w.scale)
    return compare(gpu, ref, tol, heads=heads)


# -------------------------------------------------------- fp32 I/O mode ---

def test_config1_fp32_segments():
    """fp32, B=1, H=2, T=256, d=64, C=64, two segments of 128 with state handoff."""
    w = CONFIGS["c1_f32_small"]
    inp = make_inputs(w)
    d = to_device(inp)
    gpu = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(d, w.C, w.N).items()}
    ref = oracle_fwd_bwd(inp, N=w.N)
    compare(gpu, ref, TOL_F32)
    check(w, TOL_F32)


@pytest.mark.parametrize("g_mode,g_shift", [("softplus", -4.0), ("zero", 0.0)])
def test_config1_slow_decay(g_mode, g_shift):
    """Slow decay keeps the state (and its handoff) numerically alive."""
    w = CONFIGS["c1_f32_small"].with_(g_mode=g_mode, g_shift=g_shift, S_in_std=0.05)
    check(w, TOL_F32)
    inp = make_inputs(w)
    gpu = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(to_device(inp), w.C, w.N).items()}
    compare(gpu, oracle_fwd_bwd(inp, N=w.N), TOL_F32)


@pytest.mark.parametrize("C", [16, 32, 64, 128])
@pytest.mark.parametrize("dk,dv", [(64, 64), (32, 128), (128, 16)])
def test_fp32_chunk_and_head_sizes(C, dk, dv):
    check(small(C=C, dk=dk, dv=dv, T=2 * C + 5, g_shift=-2.0), TOL_F32)


@pytest.mark.parametrize("T", [1, 15, 64, 65, 200])
def test_fp32_ragged_lengths(T):
    check(small(T=T, g_shift=-3.0), TOL_F32)


def test_fp32_beta_off_and_scale():
    check(small(use_beta=False, qk="scaled", g_shift=0.0, scale=0.125), TOL_F32)
    check(small(scale=0.5, g_mode="zero"), TOL_F32)


def test_fp32_no_states():
    check(small(S_in_std=0.0, dS_out_std=0.0, g_shift=-3.0), TOL_F32)


def test_empty_inputs():
    w = small(T=0)
    inp = to_device(make_inputs(w))
    o, S_out = sf.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S_in"], C=64)
    torch.cuda.synchronize()
    assert o.shape == (2, 3, 0, 64)
    assert torch.equal(S_out, inp["S_in"])
    gr = sf.bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S_in"], inp["dO"],
                inp["dS_out"], C=64)
    assert torch.equal(gr["dS_in"], inp["dS_out"])
    w0 = small(B=0)
    inp0 = to_device(make_inputs(w0))
    o0, _ = sf.fwd(inp0["q"], inp0["k"], inp0["v"], inp0["g"], inp0["beta"], None, C=64)
    assert o0.numel() == 0


# --------------------------------------------------------- bf16 I/O mode ---

@pytest.mark.parametrize("dk,dv,beta", [(128, 128, True), (128, 128, False), (128, 64, False), (128, 64, True),
                                        (64, 64, True)])
def test_bf16_small(dk, dv, beta):
    w = small(io="bf16", dk=dk, dv=dv, use_beta=beta, qk="l2norm" if beta else "scaled",
              g_shift=-4.0)
    check(w, TOL_BF16)


@pytest.mark.parametrize("T", [1, 17, 63])
@pytest.mark.parametrize("beta", [True, False])
def test_bf16_shorter_than_a_chunk(T, beta):
    """A sequence shorter than one chunk: no tensor map can be made, every tile
    takes the per-thread copies."""
    w = small(io="bf16", dk=128, dv=128, T=T, use_beta=beta, qk="l2norm" if beta else "scaled",
              g_shift=-4.0)
    check(w, TOL_BF16)


@pytest.mark.parametrize("C", [32, 64, 128])
def test_bf16_chunk_sizes(C):
    check(small(io="bf16", dk=128, dv=128, C=C, T=3 * C + 11, g_shift=-4.0), TOL_BF16)


def test_config2_sampled_heads():
    """bf16, B=2, H=16, T=8192, d=128, C=64, S_in ~ N(0, 0.02), N=4 segments."""
    w = CONFIGS["c2_bf16_b2h16"]
    heads = [(0, 0), (0, 7), (1, 3), (1, 15)]
    inp = make_inputs(w)
    d = to_device(inp)
    gpu = gpu_fwd_bwd(d, w.C)
    ref = oracle_fwd_bwd(inp, heads=heads)
    compare(gpu, ref, TOL_BF16, heads=heads)
    seg = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(d, w.C, w.N).items()}
    compare(seg, ref, TOL_BF16, heads=heads)


@pytest.mark.parametrize("g_mode,g_shift", [("softplus", -4.0), ("zero", 0.0)])
def test_config2_slow_decay_sampled(g_mode, g_shift):
    w = CONFIGS["c2_bf16_b2h16"].with_(g_mode=g_mode, g_shift=g_shift)
    heads = [(0, 1), (1, 10)]
    inp = make_inputs(w)
    d = to_device(inp)
    ref = oracle_fwd_bwd(inp, heads=heads)
    compare(gpu_fwd_bwd(d, w.C), ref, TOL_BF16, heads=heads)
    seg = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(d, w.C, w.N).items()}
    compare(seg, ref, TOL_BF16, heads=heads)


def test_headline_shape_sampled_heads():
    """B=1, H=16, T=65536, d=128, C=64, bf16: the benchmarked call, two heads checked."""
    w = CONFIGS["headline_h16_t64k"]
    heads = [(0, 0), (0, 11)]
    inp = make_inputs(w)
    gpu = gpu_fwd_bwd(to_device(inp), w.C)
    compare(gpu, oracle_fwd_bwd(inp, heads=heads), TOL_BF16, heads=heads)


def test_config4_beta_off_sampled_heads():
    """Scalar-gated recurrence without the delta term, H=64, T=32768, dk=128, dv=64."""
    w = CONFIGS["c4_betaoff_h64"]
    heads = [(0, 5), (0, 63)]
    inp = make_inputs(w)
    d = to_device(inp)
    ref = oracle_fwd_bwd(inp, heads=heads)
    compare(gpu_fwd_bwd(d, w.C), ref, TOL_BF16, heads=heads)
    seg = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(d, w.C, w.N).items()}
    compare(seg, ref, TOL_BF16, heads=heads)


def test_retrieval_invariant_full_size():
    """beta = 1, unit keys, q = k: o = v exactly in exact arithmetic, at the headline size."""
    w = CONFIGS["headline_h16_t64k"]
    inp = to_device(make_inputs(w))
    ones = torch.ones_like(inp["beta"])
    o, _ = sf.fwd(inp["k"], inp["k"], inp["v"], inp["g"], ones, None, C=w.C)
    torch.cuda.synchronize()
    v = inp["v"].double()
    err = (o.double() - v).abs().max().item() / v.abs().max().item()
    assert err <= TOL_BF16, err


# ----------------------------------------------------- segment identity ---

def _bit_identical(a: dict, b: dict):
    for name in a:
        if a[name] is None:
            assert b[name] is None
            continue
        assert torch.equal(a[name], b[name]), name


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_segments_bit_identical_small(io):
    w = small(io=io, dk=128 if io == "bf16" else 64, dv=128 if io == "bf16" else 64, T=8 * 64,
              g_shift=-4.0)
    d = to_device(make_inputs(w))
    one = gpu_segments(d, w.C, 1)
    for N in (2, 4, 8):
        _bit_identical(gpu_segments(d, w.C, N), one)
    _bit_identical(gpu_segments(d, w.C, 3, seg_len=[64, 320, 128]), one)
    _bit_identical(gpu_segments(d, w.C, 3, seg_len=[0, 512, 0]), one)


def test_segments_ragged_match_oracle():
    """Segment lengths that are not multiples of C: exact up to rounding."""
    w = small(io="f32", T=300, g_shift=-3.0)
    inp = make_inputs(w)
    seg_len = [37, 100, 0, 163]
    gpu = {k: None if v is None else v.double().cpu().numpy()
           for k, v in gpu_segments(to_device(inp), w.C, 4, seg_len=seg_len).items()}
    compare(gpu, oracle_fwd_bwd(inp, seg_len=seg_len), TOL_F32)


def test_config3_chain_bit_identical_and_sampled():
    """H=32, T=65536, 16 segments of 4096 (fwd over all, bwd in reverse): every
    segment count gives the same bits; one head checked against the oracle."""
    w = CONFIGS["c3_chain_h32"]
    inp = make_inputs(w)
    d = to_device(inp)
    one = gpu_segments(d, w.C, 1)
    for N in (2, 4, 8, 16):
        _bit_identical(gpu_segments(d, w.C, N), one)
    heads = [(0, 21)]
    got = {k: None if v is None else v.double().cpu().numpy() for k, v in one.items()}
    compare(got, oracle_fwd_bwd(inp, heads=heads), TOL_BF16, heads=heads)


@pytest.mark.parametrize("C", [32, 64, 128])
def test_config5_256k_bit_identical(C):
    """T=262144, H=16: N in {1,2,4,8,16} bit-identical for each chunk length."""
    w = CONFIGS["c5_256k"].with_(C=C)
    d = to_device(make_inputs(w))
    one = gpu_segments(d, C, 1)
    for N in (2, 4, 8, 16):
        _bit_identical(gpu_segments(d, C, N), one)
    for v in one.values():
        if v is not None:
            assert torch.isfinite(v.float()).all()
