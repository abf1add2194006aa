"""The delta rule with a per-channel (diagonal) decay on the GPU (through the
C ABI) against the fp64 oracle (oracle/kda.py), its split invariance, and its
reduction to the scalar-decay kernels when all channels decay alike.
Bars: max-relative error per tensor <= 1e-4 (fp32 I/O), <= 2e-2 (bf16 I/O)."""
import numpy as np
import pytest
import torch

import chunked_gated_delta_13_b200 as sf
from chunked_gated_delta_13_b200.inputs import Workload, as_f64, make_kda_inputs
from gpu_util import relerr, to_device
from oracle import kda

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
NAMES = ("o", "S_out", "dq", "dk", "dv", "dg", "dbeta", "dS_in")


def run_gpu(d, scale=1.0):
    o, S_out = sf.kda_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], scale=scale)
    gr = sf.kda_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"], d["dS_out"], scale=scale)
    torch.cuda.synchronize()
    out = {"o": o, "S_out": S_out}
    out.update(gr)
    return out


def run_oracle(inp, heads=None, scale=1.0):
    f = as_f64(inp)
    if heads is not None:
        f = {k: None if v is None else v[:, heads] for k, v in f.items()}
    o, S_out = kda.kda_fwd(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], scale)
    gr = kda.kda_bwd(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], f["dO"], f["dS_out"], scale)
    out = {"o": o, "S_out": S_out}
    out.update(gr)
    return out


def compare(gpu, ref, tol, heads=None):
    errs = {}
    for n in NAMES:
        if ref.get(n) is None:
            assert gpu.get(n) is None
            continue
        g = gpu[n].double().cpu().numpy()
        if heads is not None:
            g = g[:, heads]
        errs[n] = relerr(g, ref[n])
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"above {tol}: {bad} (all {errs})"
    return errs


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,T,beta", [(128, 128, 200, True), (64, 32, 129, True), (32, 64, 64, False),
                                          (128, 64, 1, True)])
def test_kda_matches_oracle(io, dk, dv, T, beta):
    w = Workload("kda", B=2, H=2, T=T, dk=dk, dv=dv, io=io, use_beta=beta, qk="l2norm" if beta else "scaled",
                 g_shift=-1.0, S_in_std=0.05, dS_out_std=0.1)
    inp = make_kda_inputs(w)
    compare(run_gpu(to_device(inp), 0.5), run_oracle(inp, scale=0.5), TOL[io])


def test_kda_split_invariance():
    """The state handed between two calls is the state the one-call run carries:
    every output of two segments equals the one-segment run bit for bit."""
    w = Workload("kda", B=1, H=2, T=300, dk=128, dv=128, io="bf16", g_shift=-2.0, S_in_std=0.05, dS_out_std=0.1)
    d = to_device(make_kda_inputs(w))
    one = run_gpu(d)
    cut = 117
    part = lambda x, a, b: None if x is None else x[:, :, a:b].contiguous()
    a = {n: part(d[n], 0, cut) for n in ("q", "k", "v", "g", "beta", "dO")}
    b = {n: part(d[n], cut, 300) for n in ("q", "k", "v", "g", "beta", "dO")}
    o1, S1 = sf.kda_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], d["S_in"])
    o2, S2 = sf.kda_fwd(b["q"], b["k"], b["v"], b["g"], b["beta"], S1)
    g2 = sf.kda_bwd(b["q"], b["k"], b["v"], b["g"], b["beta"], S1, b["dO"], d["dS_out"])
    g1 = sf.kda_bwd(a["q"], a["k"], a["v"], a["g"], a["beta"], d["S_in"], a["dO"], g2["dS_in"])
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], 2), one["o"]) and torch.equal(S2, one["S_out"])
    for n in ("dq", "dk", "dv", "dg", "dbeta"):
        assert torch.equal(torch.cat([g1[n], g2[n]], 2), one[n]), n
    assert torch.equal(g1["dS_in"], one["dS_in"])


def test_kda_equal_decay_matches_scalar_decay_kernels():
    """With the same log-decay on every channel the layer is the scalar-decay
    one: the per-channel kernels agree with sf_gdn_fwd / sf_gdn_bwd."""
    w = Workload("kda", B=1, H=2, T=256, dk=128, dv=128, io="f32", g_shift=-2.0, S_in_std=0.05, dS_out_std=0.1)
    inp = make_kda_inputs(w)
    gs = inp["g"][..., 0].contiguous()
    inp["g"] = gs[..., None].expand(-1, -1, -1, 128).contiguous()
    d = to_device(inp)
    a = run_gpu(d)
    o, S_out = sf.fwd(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], d["S_in"], C=64)
    gr = sf.bwd(d["q"], d["k"], d["v"], gs.cuda(), d["beta"], d["S_in"], d["dO"], d["dS_out"], C=64)
    torch.cuda.synchronize()
    b = {"o": o, "S_out": S_out, **gr}
    for n in ("o", "S_out", "dq", "dk", "dv", "dbeta", "dS_in"):
        assert relerr(a[n].double().cpu().numpy(), b[n].double().cpu().numpy()) <= 1e-4, n
    assert relerr(a["dg"].sum(-1).double().cpu().numpy(), b["dg"].double().cpu().numpy()) <= 1e-4


def test_kda_long_sequence_sampled_heads():
    """B=1, H=16, T=16384, dk=dv=128, bf16, live per-channel decay: two heads
    compared with the oracle."""
    w = Workload("kda", B=1, H=16, T=16384, dk=128, dv=128, io="bf16", g_shift=-4.0, S_in_std=0.02,
                 dS_out_std=0.1)
    inp = make_kda_inputs(w)
    heads = [5, 11]
    errs = compare(run_gpu(to_device(inp)), run_oracle(inp, heads=heads), TOL["bf16"], heads=heads)
    print("\nERRORS kda T=16384:", " ".join(f"{k}={v:.3e}" for k, v in errs.items()))
