#!/usr/bin/env python
"""Benchmark of the gated delta-rule chunk forward+backward on B200.

One step = one pass of the whole path on one batch of synthetic input:
sf_segment_run over the sequence split into N segments (forward over the
segments with the state handed on, then backward in reverse with the state
gradient handed back), i.e. UT transform, chunk scan, output with the
intra-chunk backward products, reverse state-gradient scan and the parallel
gradient kernel for every segment.  Defaults: the B=1, H=16, T=65536, d=128
workload as 16 segments, 3 warm-up and 50 timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--segments N] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is Mtokens/s of forward+backward over
all ranks (each rank runs its own independent batch: weak scaling, no
collective on the data path).  `--impl reference` times the fp64 CPU oracle on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-delta chunk fwd+bwd Mtokens/s at H=16,d=128; % of bf16 roofline"
UNIT = "Mtokens/s"
DEFAULT_WORKLOAD = "headline_h16_t64k"
DEFAULT_SEGMENTS = 16
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------ work model ----
# Algorithmic work of the method (its GEMMs, no recompute; bytes across the
# boundary with bf16 I/O and fp32 g/beta), per token per head.

def algo_flops_per_token_head(C, dk, dv, use_beta=True):
    if use_beta:
        fwd = 2 * C * (3 * dk + 2 * dv) + 6 * dk * dv
        bwd = 2 * C * (5 * dk + 4 * dv) + 12 * dk * dv
    else:
        fwd = 2 * C * (dk + dv) + 4 * dk * dv
        bwd = 2 * C * (2 * dk + 2 * dv) + 8 * dk * dv
    return fwd, bwd


def algo_bytes_per_token_head(dk, dv, esize=2, use_beta=True):
    gb = 8 if use_beta else 4
    fwd = esize * (2 * dk + dv) + gb + esize * dv
    bwd = esize * (2 * dk + dv) + gb + esize * dv + esize * (2 * dk + dv) + gb
    return fwd, bwd


def kernel_work(name, w, T_seg):
    """Work of ONE launch of kernel `name` on a segment of T_seg tokens (all
    B*H heads): (bound, algorithmic flops, algorithmic bytes, intermediate bytes).

    Algorithmic flops are the method's products the kernel contributes (no
    recompute).  Algorithmic bytes are the boundary tensors the kernel reads or
    writes (bf16 or fp32 I/O, fp32 g and beta): the state scans touch none
    per token, the gradient kernel all of the backward's (q, k, v, dO, g, beta
    in; dq, dk, dv, dg, dbeta out).  Intermediate bytes are the per-chunk
    tensors of the chunked decomposition the kernel reads or writes once (bf16
    tiles, fp32 G and L): a cost of the decomposition, reported apart and not
    credited to the roofline."""
    C, dk, dv = w.C, w.dk, w.dv
    es = 2 if w.io == "bf16" else 4
    n = w.B * w.H * T_seg                      # token-heads in the launch
    nch = w.B * w.H * ((T_seg + C - 1) // C)   # chunk-heads in the launch
    wu = 4 if name.startswith("simt") else 2   # intermediate storage bytes per element
    gb = 8 if w.use_beta else 4                # g (and beta) per token
    lb = C * C * 4 if w.use_beta else 0        # L per chunk
    state = dk * dv * wu                       # one chunk state tile
    if name.endswith("prep"):                  # k, v, g, beta -> G, exp G, -W, Khat, U^T, L
        flops = nch * (2 * C * C * dk * (2 if w.use_beta else 0) + 2 * C * C * dv * (1 if w.use_beta else 0))
        return "hbm", flops, n * (es * (dk + dv) + gb), n * (8 + wu * (2 * dk + dv)) + nch * lb
    if name.endswith("scan_fwd"):              # -W, Khat, U^T, exp G -> V_new^T, chunk states
        flops = nch * 2 * (2 * C * dk * dv)
        return "tensor", flops, 0, n * (wu * (2 * dk + dv) + 4 + wu * dv) + nch * state
    if name.endswith("scan_bwd"):              # -W, Khat, dVi^T, exp G, D^T -> dV_new^T, dS_C^T
        flops = nch * 2 * (2 * C * dk * dv)
        return "tensor", flops, 0, n * (wu * (2 * dk + dv) + 4 + wu * dv) + nch * 2 * state
    if name.endswith("out_og"):                # q, k, dO, G, V_new^T, S0^T -> o, dVi^T, D^T
        flops = nch * (2 * C * dk * dv + 2 * C * C * dk + 2 * C * C * dv) + nch * (2 * C * C * dv + 2 * C * dk * dv)
        return "hbm", flops, n * es * (2 * dk + 2 * dv), n * (4 + 2 * wu * dv) + nch * 2 * state
    if name.endswith("out"):                   # q, k, G, V_new^T, S0^T -> o
        flops = nch * (2 * C * dk * dv + 2 * C * C * dk + 2 * C * C * dv)
        return "hbm", flops, n * es * (2 * dk + dv), n * (4 + wu * dv) + nch * state
    if name.endswith("intra"):                 # q, k, dO, G -> dVi^T, D^T
        flops = nch * (2 * C * C * dk + 2 * C * C * dv + 2 * C * dk * dv)
        return "hbm", flops, n * es * (2 * dk + dv), n * (4 + wu * dv) + nch * state
    # parallel gradients: dP K, dP^T Q, dW (gamma K)^T, T^T dW, dA K (C^2 dk each),
    # dO V_new^T, dU V^T, T^T dU (C^2 dv each), dO S0^T, V_new dS^T, dV_new S0^T (C dk dv each);
    # q, k, v, dO, g, beta -> dq, dk, dv, dg, dbeta; reads V_new, dV_new, S0, dS_C, L
    flops = nch * (2 * C * C * 5 * dk + 2 * C * C * 3 * dv + 3 * 2 * C * dk * dv)
    _, abi = algo_bytes_per_token_head(dk, dv, es, w.use_beta)
    return "hbm", flops, n * abi, n * 2 * wu * dv + nch * (2 * state + lb)


def step_roofline(w, ms, pk):
    """The whole step against the binding roofline (the metric's "% of bf16
    roofline"): algorithmic flops and ABI bytes of forward + backward over every
    token-head, at the measured peaks.  `frac` is t_roof / t_step for the binding
    bound; `frac_tensor_sustained` is the step's algorithmic rate against the
    sustained bf16 peak."""
    ff, fb = algo_flops_per_token_head(w.C, w.dk, w.dv, w.use_beta)
    bf_, bb = algo_bytes_per_token_head(w.dk, w.dv, 2 if w.io == "bf16" else 4, w.use_beta)
    th = w.B * w.H * w.T
    t_flop = th * (ff + fb) / (pk["bf16_tflops"] * 1e12)
    t_hbm = th * (bf_ + bb) / (pk["hbm_gbs"] * 1e9)
    t_roof = max(t_flop, t_hbm)
    tflops = th * (ff + fb) / (ms * 1e-3) / 1e12
    return {"bound": "hbm" if t_hbm >= t_flop else "tensor", "t_roof_ms": t_roof * 1e3,
            "frac": t_roof / (ms * 1e-3), "algo_tflops": tflops,
            "algo_gbs": th * (bf_ + bb) / (ms * 1e-3) / 1e9,
            "frac_tensor_sustained": tflops / pk["bf16_tflops_sustained"]}


# DRAM bytes (read + write) per chunk-head measured by ncu
# (dram__bytes_read.sum + dram__bytes_write.sum) for each kernel of the
# tensor-core path on the small case of the headline shape (B=1, H=16, T=8192,
# d=128, one segment cut into two 4096-token pipeline pieces: 1024 chunk-heads
# per launch, one launch of the timed step).  A launch's traffic is this figure
# times its chunk-heads.  Valid for the kernels as they were when
# captured; an entry is removed when its kernel changes.
MEASURED_TRAFFIC = {
    "tc_prep": 45119.0,
    "tc_scan_fwd": 60996.0,
    "tc_out_og": 123340.0,
    "tc_scan_bwd": 102798.0,
    "tc_grad": 206943.0,
}


# ---------------------------------------------------------------- helpers ---

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_workload(name, rank, chunk=0):
    """Replicas: every rank runs its own independent batch, the named workload
    with the seed offset by the rank (no data crosses ranks); `chunk` > 0
    overrides the kernel chunk length."""
    from chunked_gated_delta_13_b200.inputs import CONFIGS
    w = CONFIGS[name]
    if chunk:
        w = w.with_(C=chunk)
    return w.with_(seed=w.seed + rank)


def max_over_ranks(x, ws, device):
    """The slowest rank's value of x (all ranks take part; a no-op on one rank)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_mtokens_per_s(tokens_per_rank, ws, ms):
    """Whole-job throughput: the tokens all ranks processed over the step time
    (already the maximum over ranks)."""
    return tokens_per_rank * ws / (ms * 1e-3) / 1e6


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.idx = device_index
        self.lines = []
        self.mark_at = None
        self.thread = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return

        def reader():
            for line in self.proc.stdout:
                self.lines.append(line)

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def mark(self, wait_s=5.0):
        """Call just before the timed region: waits for the sampler's first line,
        then remembers where the timed region's samples begin."""
        t = time.time()
        while self.proc is not None and not self.lines and time.time() - t < wait_s:
            time.sleep(0.01)
        self.mark_at = len(self.lines)

    def stop(self):
        if self.proc is None:
            return None
        timed = len(self.lines) - (self.mark_at or 0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        # the samples taken during the timed region, else (region shorter than
        # the sampling interval) all samples of the run
        lines = self.lines[self.mark_at:self.mark_at + timed] if self.mark_at is not None and timed > 0 \
            else self.lines
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "in_timed_region": bool(self.mark_at is not None and timed > 0)}


# --------------------------------------------------------- reference arm ---

def run_reference(args):
    """Time the fp64 CPU oracle (as it stands) on a bounded sample of the workload."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401
    import oracle
    from chunked_gated_delta_13_b200.inputs import CONFIGS, as_f64, make_inputs

    w = CONFIGS[args.workload]
    if args.chunk:
        w = w.with_(C=args.chunk)
    seg = args.segments if args.segments else w.N
    budget_s = float(os.environ.get("SF_REF_STEP_SECONDS", "1.5"))

    def sample_inputs(T):
        f = as_f64(make_inputs(w.with_(T=T)))
        return f

    def one_step(f, T):
        N = max(1, min(seg, T // w.C)) if T >= w.C else 1
        oracle.segment_run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], f["dO"],
                           f["dS_out"], N=N)

    # calibrate the T-prefix so that one step takes about `budget_s`
    T_cal = min(w.T, 256)
    f = sample_inputs(T_cal)
    t = time.perf_counter()
    one_step(f, T_cal)
    dt = time.perf_counter() - t
    T_s = int(max(w.C, min(w.T, T_cal * budget_s / max(dt, 1e-6))) // w.C * w.C)
    f = sample_inputs(T_s)
    for _ in range(args.warmup):
        one_step(f, T_s)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        one_step(f, T_s)
        times.append(time.perf_counter() - t)
    per = sum(times) / len(times)
    value = w.B * T_s / per / 1e6
    sample = (f"{w.B}x{w.H} heads x first {T_s} of {w.T} tokens (fp64, fwd+bwd, "
              f"{min(seg, max(1, T_s // w.C))} segments); cost is linear in tokens")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": T_s, "T_full": w.T, "dk": w.dk,
                   "dv": w.dv, "C": w.C, "segments": seg},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(w, seg, seconds=15.0):
    """The oracle on a bounded T-prefix of the workload, all heads (rank 0, N=1)."""
    import oracle
    from chunked_gated_delta_13_b200.inputs import as_f64, make_inputs
    T_cal = min(w.T, 256)
    f = as_f64(make_inputs(w.with_(T=T_cal)))
    t = time.perf_counter()
    oracle.segment_run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], f["dO"], f["dS_out"],
                       N=1)
    dt = time.perf_counter() - t
    T_s = int(max(w.C, min(w.T, T_cal * seconds / max(dt, 1e-6))) // w.C * w.C)
    f = as_f64(make_inputs(w.with_(T=T_s)))
    N = max(1, min(seg, T_s // w.C))
    t = time.perf_counter()
    oracle.segment_run(f["q"], f["k"], f["v"], f["g"], f["beta"], f["S_in"], f["dO"], f["dS_out"],
                       N=N)
    dt = time.perf_counter() - t
    return {"value": w.B * T_s / dt / 1e6, "unit": UNIT, "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"{w.B}x{w.H} heads x first {T_s} of {w.T} tokens, fp64 fwd+bwd, "
                      f"{N} segments, {dt:.1f} s"}


# ---------------------------------------------------------------- our arm ---

def run_ours(args):
    import torch
    import torch.distributed as dist

    import chunked_gated_delta_13_b200 as sf
    from chunked_gated_delta_13_b200.inputs import CONFIGS, make_inputs

    ws, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", rank=rank, world_size=ws,
                                timeout=datetime.timedelta(seconds=120), device_id=dev)

    w = rank_workload(args.workload, rank, args.chunk)
    seg = args.segments if args.segments else w.N
    inp_cpu = make_inputs(w)
    d = {k: None if v is None else v.to(dev).contiguous() for k, v in inp_cpu.items()}
    shape = sf.make_shape(w.B, w.H, w.T, w.dk, w.dv, w.C, w.io, w.use_beta, w.scale)
    stream = torch.cuda.current_stream(dev)
    nbytes = sf.segment_workspace_bytes(shape, seg)
    wsbuf = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    out = {"o": torch.empty_like(d["v"]),
           "S_out": torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=dev),
           "dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]),
           "dv": torch.empty_like(d["v"]),
           "dg": torch.empty(w.B, w.H, w.T, dtype=torch.float32, device=dev),
           "dbeta": None if d["beta"] is None else torch.empty_like(d["beta"]),
           "dS_in": torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=dev)}

    def step(src=d, dst=out):
        sf.segment_run(src["q"], src["k"], src["v"], src["g"], src["beta"], src["S_in"], src["dO"],
                       src["dS_out"], N=seg, C=w.C, scale=w.scale, out=dst, workspace=wsbuf,
                       stream=stream)

    def barrier():
        if ws > 1:
            dist.barrier()

    def max_ranks(x):
        return max_over_ranks(x, ws, dev)

    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # per-kernel timing: the library records a CUDA event pair around each of
    # its launches on the launch's own stream (native, a few microseconds of
    # host time per launch, so the timed steps are not slowed by the probe);
    # one extra untimed step counts the launches per step
    sf.timer_enable(1 << 14)
    step()
    torch.cuda.synchronize(dev)
    per_step_launches = sf.timer_count()
    sf.timer_enable(per_step_launches * args.steps)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.mark()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    sf.timer_disable()
    ms = t0.elapsed_time(t1) / args.steps
    ms = max_ranks(ms)
    clk = clocks.stop()

    # per-kernel durations inside the timed region
    per = {}
    for name, dur in sf.timer_results():
        per.setdefault(name, []).append(dur)
    sf.timer_free()
    launches = sum(len(v) for v in per.values()) // args.steps

    # end-to-end: every step copies its inputs from pinned host memory to the
    # device and all its results back to pinned host memory, inside the timed
    # region.  Two device sets of inputs and results and two copy streams
    # (PCIe is full duplex) let step k+1's input copy and step k-1's result
    # copy run while step k computes, as a training loop that prefetches its
    # next batch would.
    pin = {k: None if v is None else v.pin_memory() for k, v in inp_cpu.items()}
    host_out = {k: None if v is None else torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                for k, v in out.items()}
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in host_out.values() if v is not None)
    dsets = [{k: None if v is None else torch.empty_like(v) for k, v in d.items()} for _ in range(2)]
    osets = [out, {k: None if v is None else torch.empty_like(v) for k, v in out.items()}]
    h2d_s = torch.cuda.Stream(dev)
    d2h_s = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n, start_event):
        h2d_s.wait_event(start_event)
        for k in range(n):
            b = k % 2
            with torch.cuda.stream(h2d_s):
                if k >= 2:
                    h2d_s.wait_event(ev_done[b])  # step k-2 has read this input set
                for name, v in pin.items():
                    if v is not None:
                        dsets[b][name].copy_(v, non_blocking=True)
                ev_in[b].record(h2d_s)
            stream.wait_event(ev_in[b])
            if k >= 2:
                stream.wait_event(ev_out[b])  # step k-2's results are back on the host
            step(dsets[b], osets[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[b])
                for name, v in osets[b].items():
                    if v is not None:
                        host_out[name].copy_(v, non_blocking=True)
                ev_out[b].record(d2h_s)
        stream.wait_event(ev_out[(n - 1) % 2])

    w0 = torch.cuda.Event()
    w0.record(stream)
    e2e_run(2, w0)
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(2, min(args.steps, 6))
    e0.record(stream)
    e2e_run(n_e2e, e0)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_ranks(e0.elapsed_time(e1) / n_e2e)

    value = job_mtokens_per_s(w.B * w.T, ws, ms)
    pk = peaks()

    # roofline of the dominant kernel
    tot = {k: sum(v) for k, v in per.items()}
    dom = max(tot, key=tot.get) if tot else None
    roof = None
    if dom:
        # the library cuts segments into pipeline pieces, so a launch covers a
        # share of the step: per-launch work = the step's work / launches per step
        per_step = len(per[dom]) / args.steps
        T_seg = -(-w.T // seg)
        bound, flops, byts, inter = kernel_work(dom, w, T_seg)
        flops, byts, inter = (x * seg / per_step for x in (flops, byts, inter))
        avg_ms = tot[dom] / len(per[dom])
        nch_launch = w.B * w.H * (-(-T_seg // w.C)) * seg / per_step
        traffic = (MEASURED_TRAFFIC[dom] * nch_launch if dom in MEASURED_TRAFFIC and w.io == "bf16"
                   and w.dk == 128 and w.dv == 128 and w.C == 64 else None)
        if bound == "hbm":
            ach = byts / (avg_ms * 1e-3) / 1e9
            peak = pk["hbm_gbs"]
            unit = "GB/s"
        else:
            ach = flops / (avg_ms * 1e-3) / 1e12
            peak = pk["bf16_tflops_sustained"]
            unit = "TFLOP/s"
        roof = {"bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
                "traffic": traffic, "kernel": dom, "avg_launch_ms": avg_ms,
                "algorithmic_bytes": byts, "algorithmic_flops": flops,
                "intermediate_bytes": inter,
                "waste": (traffic / byts) if (traffic is not None and byts > 0) else None,
                "share": tot[dom] / sum(tot.values()), "peak_source": pk["source"]}

    step_roof = step_roofline(w, ms, pk)

    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(w.with_(seed=CONFIGS[args.workload].seed), seg)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.io, "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "dk": w.dk, "dv": w.dv,
                       "C": w.C, "segments": seg, "path": sf.path(shape),
                       "parallelism": f"replicas x{ws} (independent batches)",
                       "l2": (f"inputs {sum(v.numel() * v.element_size() for v in d.values() if v is not None) / 2**20:.0f} MiB"
                              f" > L2 {L2_BYTES / 2**20:.0f} MiB, no flush")},
            "roofline": roof, "roofline_step": step_roof,
            "kernels_ms": {k: {"launches": len(v), "total_ms": sum(v), "share": sum(v) / sum(tot.values())}
                           for k, v in per.items()},
            "cpu_baseline": cpu,
            "e2e": {"value": job_mtokens_per_s(w.B * w.T, ws, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--segments", type=int, default=DEFAULT_SEGMENTS)
    ap.add_argument("--chunk", type=int, default=0, help="kernel chunk length C (0 = the workload's)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
