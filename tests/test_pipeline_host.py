"""The multi-rank sequence pipeline (chunked_gated_delta_13_b200.pipeline) on
the CPU: its schedule keeps the dependency order and cannot deadlock, and two
or three gloo ranks, each computing its segment with the fp64 oracle, give
exactly the single-process segment chain's results for every microbatch."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from chunked_gated_delta_13_b200 import pipeline  # noqa: E402


@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("M", [0, 1, 2, 5, 9])
def test_schedule_order_and_no_deadlock(P, M):
    for r in range(P):
        order = pipeline.schedule(P, M, r)
        assert sorted(order) == sorted([("F", a) for a in range(M)] + [("B", a) for a in range(M)])
        for a in range(M):
            assert order.index(("F", a)) < order.index(("B", a))
        fwd = [a for k, a in order if k == "F"]
        assert fwd == sorted(fwd)
        # at most P - r microbatches are between their forward and backward at once
        live = peak = 0
        for k, _ in order:
            live += 1 if k == "F" else -1
            peak = max(peak, live)
        assert peak <= max(1, min(M, P - r))
    pipeline.check_schedule(P, M)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_stage():
    import torch

    import oracle

    class OracleStage(pipeline.Stage):
        """Segment arithmetic with the fp64 oracle (test infrastructure)."""

        def __init__(self):
            self.saved = {}

        def new_state(self, seg):
            B, H, _, dk = seg.q.shape
            return torch.empty(B, H, dk, seg.v.shape[-1], dtype=torch.float64)

        def fwd(self, a, seg, S_in):
            n = lambda t: None if t is None else t.numpy()
            o, S_out = oracle.gdn_fwd(n(seg.q), n(seg.k), n(seg.v), n(seg.g), n(seg.beta), n(S_in))
            self.saved[a] = S_in
            return torch.from_numpy(o), torch.from_numpy(np.ascontiguousarray(S_out))

        def bwd(self, a, seg, dS_out):
            n = lambda t: None if t is None else t.numpy()
            S_in = self.saved.pop(a)
            gr = oracle.gdn_bwd(n(seg.q), n(seg.k), n(seg.v), n(seg.g), n(seg.beta), n(S_in), n(seg.dO),
                                n(dS_out))
            out = {k: None if v is None else torch.from_numpy(np.ascontiguousarray(v)) for k, v in gr.items()}
            return out, out["dS_in"]

    return OracleStage()


def _inputs(M, P, seglen):
    from chunked_gated_delta_13_b200.inputs import Workload, as_f64, make_inputs
    mbs = []
    for a in range(M):
        w = Workload("pipe", B=1, H=2, T=P * seglen, dk=8, dv=8, C=64, io="f32", S_in_std=0.1,
                     dS_out_std=0.1, g_shift=-3.0, seed=a)
        mbs.append(as_f64(make_inputs(w)))
    return mbs


def _worker(rank, ws, port, M, seglen, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        segs = []
        for f in _inputs(M, ws, seglen):
            sl = slice(rank * seglen, (rank + 1) * seglen)
            t = lambda x: None if x is None else torch.from_numpy(np.ascontiguousarray(x))
            segs.append(pipeline.SegmentData(
                q=t(f["q"][:, :, sl]), k=t(f["k"][:, :, sl]), v=t(f["v"][:, :, sl]), g=t(f["g"][:, :, sl]),
                beta=t(f["beta"][:, :, sl]), dO=t(f["dO"][:, :, sl]),
                S_in=t(f["S_in"]) if rank == 0 else None, dS_out=t(f["dS_out"]) if rank == ws - 1 else None))
        trace = []
        res = pipeline.run_pipeline(_oracle_stage(), segs, on_task=lambda k, a: trace.append((k, a)))
        out = []
        for a, r in enumerate(res):
            rec = {"o": r["o"].numpy()}
            rec.update({k: None if v is None else v.numpy() for k, v in r["grads"].items() if k != "dS_in"})
            if "dS_in" in r:
                rec["dS_in"] = r["dS_in"].numpy()
            if "S_out" in r:
                rec["S_out"] = r["S_out"].numpy()
            out.append(rec)
        queue.put((rank, out, trace))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2, 3])
def test_pipeline_over_gloo_matches_the_segment_chain(ws):
    import oracle
    M, seglen = 3, 20
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, M, seglen, queue)) for r in range(ws)]
    for p in procs:
        p.start()
    try:
        got = {}
        for _ in procs:
            rank, out, trace = queue.get(timeout=300)
            got[rank] = (out, trace)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in range(ws):
        assert got[r][1] == pipeline.schedule(ws, M, r)
    for a, f in enumerate(_inputs(M, ws, seglen)):
        o, S_out, gr = oracle.segment_run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], f["dO"],
                                          f["dS_out"], N=ws)
        for r in range(ws):
            rec = got[r][0][a]
            sl = slice(r * seglen, (r + 1) * seglen)
            np.testing.assert_allclose(rec["o"], o[:, :, sl], rtol=0, atol=1e-12)
            for k in ("dq", "dk", "dv", "dg", "dbeta"):
                np.testing.assert_allclose(rec[k], gr[k][:, :, sl], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[ws - 1][0][a]["S_out"], S_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[0][0][a]["dS_in"], gr["dS_in"], rtol=0, atol=1e-12)
