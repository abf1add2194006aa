"""Multi-rank plumbing of bench.py on the CPU (gloo, world size 2).

The path shards into independent replicas (one batch per rank, no data-path
collective); the only exchange is the reduction that makes every timing the
slowest rank's.  These tests run that logic as two real processes.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from chunked_gated_delta_13_b200.inputs import make_inputs

    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload("c1_f32_small", rank)
        inp = make_inputs(w)
        slowest = bench.max_over_ranks(1.5 * (rank + 1), ws, torch.device("cpu"))
        queue.put((rank, w.seed, float(inp["q"].double().sum()), slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_and_slowest_rank_timing_over_gloo():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(queue.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (r0, seed0, sum0, max0), (r1, seed1, sum1, max1) = got
    assert (r0, r1) == (0, 1)
    assert seed1 == seed0 + 1 and sum0 != sum1     # independent batches
    assert max0 == max1 == 3.0                      # every rank reports the slowest rank's time


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert abs(bench.job_mtokens_per_s(65536, 2, 4.0) - 2 * 65536 / 4e-3 / 1e6) < 1e-9
    assert bench.max_over_ranks(2.5, 1, None) == 2.5


def test_reference_arm_runs_on_rank_zero_only():
    """`bench.py --impl reference` under torchrun with two ranks: rank 0 times the
    oracle and prints the one JSON line, rank 1 exits 0 without work."""
    env = dict(os.environ, SF_REF_STEP_SECONDS="0.05", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--workload", "c1_f32_small", "--segments", "2", "--gpus", "2",
           "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [line for line in out.stdout.splitlines() if line.startswith("{")]
    assert len(lines) == 1, out.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"


def test_step_roofline_headline_figures():
    """The headline step's bound: 8.39 MFLOP and 45.4 KB per token (all 16
    heads) of algorithmic work, HBM binding at 0.46 ms per step on the measured
    peaks."""
    sys.path.insert(0, ROOT)
    import bench
    from chunked_gated_delta_13_b200.inputs import CONFIGS
    w = CONFIGS["headline_h16_t64k"]
    pk = {"hbm_gbs": 6452.5, "bf16_tflops": 1667.9, "bf16_tflops_sustained": 1378.8}
    r = bench.step_roofline(w, 4.0, pk)
    ff, fb = bench.algo_flops_per_token_head(w.C, w.dk, w.dv)
    bf_, bb = bench.algo_bytes_per_token_head(w.dk, w.dv)
    assert abs((ff + fb) * w.H / 1e6 - 8.389) < 0.01
    assert abs((bf_ + bb) * w.H / 1e3 - 45.44) < 0.01
    assert r["bound"] == "hbm" and abs(r["t_roof_ms"] - 0.4615) < 0.001
    assert abs(r["frac"] - r["t_roof_ms"] / 4.0) < 1e-12
    assert abs(r["frac_tensor_sustained"] - r["algo_tflops"] / 1378.8) < 1e-12


def test_dominant_kernel_credits_boundary_bytes_only():
    """The per-kernel roofline credits a kernel with the boundary tensors it
    moves: the gradient kernel with all of the backward's (1808 B per token-head
    at d = 128, bf16), the state scans with none; the decomposition's
    intermediates are reported apart."""
    sys.path.insert(0, ROOT)
    import bench
    from chunked_gated_delta_13_b200.inputs import CONFIGS
    w = CONFIGS["headline_h16_t64k"]
    th = w.B * w.H * 4096
    bound, flops, abi, inter = bench.kernel_work("tc_grad", w, 4096)
    assert bound == "hbm" and abi == th * 1808 and inter > 0
    _, bwd = bench.algo_bytes_per_token_head(w.dk, w.dv, 2, True)
    assert bwd == 1808
    for name in ("tc_scan_fwd", "tc_scan_bwd"):
        bound, flops, abi, inter = bench.kernel_work(name, w, 4096)
        assert bound == "tensor" and abi == 0 and flops == w.B * w.H * 64 * 2 * (2 * 64 * 128 * 128)
