"""The pipelined segment chain of the tensor-core path (sf_segment_run with bf16
I/O, dk = 128): it must compute exactly what the standalone calls compute,
run the benchmarked configuration correctly, and handle a forward-only call.
"""
import pytest
import torch

import chunked_gated_delta_13_b200 as sf
from chunked_gated_delta_13_b200.inputs import CONFIGS, Workload, make_inputs
from gpu_util import compare, gpu_fwd_bwd, oracle_fwd_bwd, to_device

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _run_segments(d, C, N, seg_len=None):
    o, S_out, gr = sf.segment_run(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"],
                                  d["dS_out"], N=N, seg_len=seg_len, C=C)
    torch.cuda.synchronize()
    sf.device_check()
    out = {"o": o, "S_out": S_out}
    out.update(gr)
    return out


def _run_calls(d, C):
    o, S_out = sf.fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], C=C)
    gr = sf.bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"], d["dS_out"], C=C)
    torch.cuda.synchronize()
    sf.device_check()
    out = {"o": o, "S_out": S_out}
    out.update(gr)
    return out


@pytest.mark.parametrize("dv,beta,T", [(128, True, 6 * 64), (128, True, 5 * 64 + 40),
                                       (64, True, 4 * 64), (64, False, 3 * 64 + 7),
                                       (128, False, 4 * 64)])
def test_pipeline_bit_identical_to_standalone_calls(dv, beta, T):
    """One-segment chain (fused Out + OG, kept intermediates, no second Pre or
    forward recompute) against sf_gdn_fwd + sf_gdn_bwd: every output bit-equal."""
    w = Workload(name="pipe", B=2, H=3, T=T, dk=128, dv=dv, C=64, io="bf16", use_beta=beta,
                 S_in_std=0.05, dS_out_std=0.1, g_shift=-4.0)
    d = to_device(make_inputs(w))
    a = _run_segments(d, w.C, 1)
    b = _run_calls(d, w.C)
    for name, x in b.items():
        if x is None:
            assert a.get(name) is None, name
            continue
        assert torch.equal(a[name], x), name


def test_headline_segment_chain_sampled_heads():
    """The benchmarked configuration: B=1, H=16, T=65536, d=128 as 16 segments,
    two heads checked against the oracle."""
    w = CONFIGS["headline_h16_t64k"]
    heads = [(0, 3), (0, 14)]
    inp = make_inputs(w)
    out = _run_segments(to_device(inp), w.C, 16)
    gpu = {k: None if v is None else v.double().cpu().numpy() for k, v in out.items()}
    compare(gpu, oracle_fwd_bwd(inp, heads=heads), TOL_BF16, heads=heads)


def test_segment_chain_forward_only():
    """dO = NULL runs the forward chain alone; its outputs equal those of a full run."""
    w = Workload(name="fwd_only", B=1, H=4, T=8 * 64, dk=128, dv=128, C=64, io="bf16",
                 S_in_std=0.05, g_shift=-4.0)
    d = to_device(make_inputs(w))
    o, S_out, gr = sf.segment_run(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], None, N=4, C=w.C)
    torch.cuda.synchronize()
    sf.device_check()
    assert gr is None
    full = _run_segments(d, w.C, 4)
    assert torch.equal(o, full["o"]) and torch.equal(S_out, full["S_out"])


def test_native_launch_timer():
    """sf_timer_*: one record per launch, named after the kernel, with a positive duration."""
    w = Workload(name="timer", B=1, H=2, T=3 * 64, dk=128, dv=128, C=64, io="bf16")
    d = to_device(make_inputs(w))
    sf.timer_enable(64)
    _run_segments(d, w.C, 1)
    sf.timer_disable()
    rec = sf.timer_results()
    sf.timer_free()
    names = [n for n, _ in rec]
    assert names == ["tc_prep", "tc_scan_fwd", "tc_out_og", "tc_scan_bwd", "tc_grad"], names
    assert all(ms > 0 for _, ms in rec)


@pytest.mark.parametrize("dv,beta,T,N", [(128, True, 6 * 64, 2), (64, False, 5 * 64 + 40, 3),
                                         (128, True, 9000, 3)])
def test_bounded_memory_chain_bit_identical(dv, beta, T, N):
    """The bounded-memory mode (boundary states only, each segment's backward
    recomputing its forward) gives the same bits as the pipelined mode."""
    w = Workload(name="bounded", B=1, H=3, T=T, dk=128, dv=dv, C=64, io="bf16", use_beta=beta,
                 S_in_std=0.05, dS_out_std=0.1, g_shift=-4.0)
    d = to_device(make_inputs(w))
    seg = [T // N // 64 * 64] * (N - 1)
    seg.append(T - sum(seg))
    a = _run_segments(d, w.C, N, seg_len=seg)
    o, S_out, gr = sf.segment_run(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"],
                                  d["dS_out"], N=N, seg_len=seg, C=w.C, bounded_memory=True)
    torch.cuda.synchronize()
    sf.device_check()
    b = {"o": o, "S_out": S_out}
    b.update(gr)
    for name, x in b.items():
        if x is None:
            assert a.get(name) is None, name
            continue
        assert torch.equal(a[name], x), name


def test_bounded_memory_headline_chain():
    """The headline chain (B=1, H=16, T=65536, d=128, 16 segments) in the
    bounded-memory mode: bit-identical to the pipelined mode."""
    w = CONFIGS["headline_h16_t64k"].with_(S_in_std=0.02, g_mode="softplus", g_shift=-4.0)
    d = to_device(make_inputs(w))
    a = _run_segments(d, w.C, 16)
    o, S_out, gr = sf.segment_run(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S_in"], d["dO"],
                                  d["dS_out"], N=16, C=w.C, bounded_memory=True)
    torch.cuda.synchronize()
    sf.device_check()
    assert torch.equal(a["o"], o) and torch.equal(a["S_out"], S_out)
    for name, x in gr.items():
        if x is not None:
            assert torch.equal(a[name], x), name


def test_rank_pipeline_cuda_stage_single_rank():
    """The multi-rank sequence pipeline with the CUDA segment arithmetic, on the
    one GPU a run here has (world size 1, NCCL): every microbatch's outputs are
    bit-identical to the standalone calls.  Two or more ranks are covered on the
    CPU (gloo, oracle arithmetic) in the host tests."""
    import datetime
    import os

    import torch.distributed as dist

    from chunked_gated_delta_13_b200 import pipeline
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29517")
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        segs, refs = [], []
        for a in range(2):
            w = Workload(name="ranks", B=1, H=2, T=5 * 64 + 9, dk=128, dv=128, C=64, io="bf16",
                         S_in_std=0.05, dS_out_std=0.1, g_shift=-4.0, seed=a)
            d = to_device(make_inputs(w))
            segs.append(pipeline.SegmentData(q=d["q"], k=d["k"], v=d["v"], g=d["g"], beta=d["beta"], dO=d["dO"],
                                             S_in=d["S_in"], dS_out=d["dS_out"]))
            refs.append(_run_calls(d, 64))
        res = pipeline.run_pipeline(pipeline.CudaStage(C=64), segs)
        torch.cuda.synchronize()
        for r, ref in zip(res, refs):
            assert torch.equal(r["o"], ref["o"]) and torch.equal(r["S_out"], ref["S_out"])
            for name in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
                assert torch.equal(r["grads"][name], ref[name]), name
            assert torch.equal(r["dS_in"], ref["dS_in"])
    finally:
        dist.destroy_process_group()
