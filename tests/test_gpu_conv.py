"""The short causal convolution with its boundary state on the GPU (called
through the C ABI) against the fp64 oracle, and the bit identity of its
segment chain.  Bars as for the recurrence: max-relative error per tensor
<= 1e-4 with fp32 I/O and <= 2e-2 with bf16 I/O."""
import numpy as np
import pytest
import torch

import chunked_gated_delta_13_b200 as sf
from chunked_gated_delta_13_b200.inputs import ConvWorkload, make_conv_inputs
from gpu_util import relerr
from oracle import shortconv as sc

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def dev(inp):
    return {k: None if v is None else v.cuda().contiguous() for k, v in inp.items()}


def oracle_all(inp, act, N=1, seg_len=None):
    f = {k: f64(v) for k, v in inp.items()}
    y, co, g = sc.segment_run(f["x"], f["w"], f["conv_in"], f["dy"], f["dconv_out"], N=N,
                              seg_len=seg_len, act=act)
    return {"y": y, "conv_out": co, **g}


def check(got, ref, tol, heads=None):
    errs = {}
    for name, r in ref.items():
        g = got[name]
        if heads is not None and name not in ("dw",):
            g = g[:, heads]
            r = r[:, heads]
        errs[name] = relerr(g, r)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"above {tol}: {bad} (all {errs})"
    return errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("act", ["silu", "none"])
@pytest.mark.parametrize("T,K,d", [(1, 4, 32), (63, 4, 128), (64, 2, 64), (200, 4, 128), (513, 3, 16)])
def test_conv_calls_match_oracle(io, act, T, K, d):
    w = ConvWorkload("c", B=2, H=3, T=T, d=d, K=K, io=io, act=act)
    inp = make_conv_inputs(w)
    d_ = dev(inp)
    y, co = sf.conv_fwd(d_["x"], d_["w"], d_["conv_in"], act=act)
    gr = sf.conv_bwd(d_["x"], d_["w"], d_["conv_in"], d_["dy"], d_["dconv_out"], act=act)
    torch.cuda.synchronize()
    got = {"y": f64(y), "conv_out": f64(co), "dx": f64(gr["dx"]), "dw": f64(gr["dw"]),
           "dconv_in": f64(gr["dconv_in"])}
    check(got, oracle_all(inp, act), TOL[io])


def test_conv_without_state_and_dw_accumulation():
    """conv_in = NULL is a zero state; dw_in is added to this segment's weight gradient."""
    w = ConvWorkload("c", B=1, H=2, T=130, d=64, K=4, io="f32", with_state=False)
    inp = make_conv_inputs(w)
    d_ = dev(inp)
    base = torch.randn(2, 64, 4, device="cuda")
    gr = sf.conv_bwd(d_["x"], d_["w"], None, d_["dy"], None, dw_in=base)
    torch.cuda.synchronize()
    ref = oracle_all(inp, "silu")
    assert relerr(f64(gr["dw"]), ref["dw"] + f64(base)) <= 1e-4


def _segments(d_, act, N, seg_len=None):
    y, co, g = sf.conv_segment_run(d_["x"], d_["w"], d_["conv_in"], d_["dy"], d_["dconv_out"], N=N,
                                   seg_len=seg_len, act=act)
    torch.cuda.synchronize()
    return {"y": y, "conv_out": co, **g}


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_segment_chain_bit_identical(io):
    """y, conv_out, dx, dconv_in are bit-identical for any split; dw too when
    every segment length is a multiple of 64."""
    w = ConvWorkload("c", B=2, H=2, T=640, d=128, K=4, io=io)
    inp = make_conv_inputs(w)
    d_ = dev(inp)
    one = _segments(d_, "silu", 1)
    for N, lens in ((2, None), (5, None), (3, [64, 512, 64]), (4, [0, 128, 0, 512])):
        got = _segments(d_, "silu", N, lens)
        for k in one:
            assert torch.equal(got[k], one[k]), (N, lens, k)
    ragged = _segments(d_, "silu", 4, [3, 1, 200, 436])
    for k in ("y", "conv_out", "dx", "dconv_in"):
        assert torch.equal(ragged[k], one[k]), k
    ref = oracle_all(inp, "silu")
    check({k: f64(v) for k, v in ragged.items()}, ref, TOL[io])
    check({k: f64(v) for k, v in one.items()}, ref, TOL[io])


def test_conv_full_size_sampled_heads():
    """The convolution of one of q, k, v at B=1, H=16, T=65536, d=128, K=4, bf16,
    as 16 segments; two heads compared with the oracle."""
    w = ConvWorkload("c", B=1, H=16, T=65536, d=128, K=4, io="bf16")
    inp = make_conv_inputs(w)
    d_ = dev(inp)
    got = _segments(d_, "silu", 16)
    heads = [3, 12]
    sub = {k: (v[:, heads].contiguous() if (v is not None and k != "w") else v) for k, v in inp.items()}
    sub["w"] = inp["w"][heads].contiguous()
    ref = oracle_all(sub, "silu")
    for k in ("y", "conv_out", "dx", "dconv_in"):
        assert relerr(f64(got[k])[:, heads], ref[k]) <= TOL["bf16"], k
    # dw sums over the batch only, so the two heads' rows are exact samples
    assert relerr(f64(got["dw"])[heads], ref["dw"]) <= TOL["bf16"]
