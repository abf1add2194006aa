"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import numpy as np
import torch

import chunked_gated_delta_13_b200 as sf
import oracle
from chunked_gated_delta_13_b200.inputs import as_f64

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dS_in")


def relerr(x, y) -> float:
    """Max-relative error of a tensor: max|x - y| / max|y| (max|x| when y == 0)."""
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    if x.size == 0:
        return 0.0
    den = float(np.max(np.abs(y)))
    num = float(np.max(np.abs(x - y)))
    return num / den if den > 0 else num


def to_device(inp: dict, device="cuda") -> dict:
    return {k: None if v is None else v.to(device).contiguous() for k, v in inp.items()}


def host(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def gpu_fwd_bwd(d: dict, C: int, scale=1.0) -> dict:
    o, S_out = sf.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], C=C, scale=scale)
    gr = sf.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"], d["dS_out"],
                C=C, scale=scale)
    torch.cuda.synchronize()
    sf.device_check()
    out = {"o": host(o), "S_out": host(S_out)}
    out.update({k: host(v) for k, v in gr.items()})
    return out


def gpu_segments(d: dict, C: int, N: int, seg_len=None, scale=1.0) -> dict:
    o, S_out, gr = sf.segment_run(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"],
                                  d["dS_out"], N=N, seg_len=seg_len, C=C, scale=scale)
    torch.cuda.synchronize()
    sf.device_check()
    out = {"o": o.clone(), "S_out": S_out.clone()}
    out.update({k: None if v is None else v.clone() for k, v in gr.items()})
    return out


def _sel(a, heads):
    if a is None or heads is None:
        return a
    return np.stack([a[b, h] for (b, h) in heads])[:, None]


def oracle_fwd_bwd(inp_cpu: dict, heads=None, scale=1.0, N=None, seg_len=None) -> dict:
    """fp64 oracle on the (b, h) pairs in `heads` (all when None); heads are
    independent, so a subset is an exact sample of the full problem."""
    f = as_f64(inp_cpu)
    s = {k: _sel(v, heads) for k, v in f.items()}
    if N is None and seg_len is None:
        o, S_out = oracle.gdn_fwd(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S_in"], scale)
        gr = oracle.gdn_bwd(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S_in"], s["dO"],
                            s["dS_out"], scale)
    else:
        o, S_out, gr = oracle.segment_run(s["q"], s["k"], s["v"], s["g"], s["beta"], s["S_in"],
                                          s["dO"], s["dS_out"], N=N, seg_len=seg_len, scale=scale)
    out = {"o": o, "S_out": S_out}
    out.update(gr)
    return out


def compare(gpu: dict, ref: dict, tol: float, heads=None, names=None):
    """Assert max-relative error <= tol for every output tensor; returns the errors."""
    errs = {}
    for name in names or (("o", "S_out") + GRADS):
        r = ref.get(name)
        g = gpu.get(name)
        if r is None:
            assert g is None or name == "dbeta", name
            continue
        g = _sel(g, heads)
        assert g.shape == r.shape, (name, g.shape, r.shape)
        assert np.all(np.isfinite(g)), f"{name}: non-finite values"
        errs[name] = relerr(g, r)
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, f"max-relative error above {tol}: {bad} (all: {errs})"
    return errs
