"""Sequence pipeline across ranks: the gated delta-rule layer of a long sequence
split into P contiguous segments, segment r on rank r (one process per GPU),
with the fp32 recurrent state handed from rank to rank and its gradient handed
back (StateFlow, arXiv 2608.06838, section 3.1).

Each microbatch a is one sequence; F(r, a) and B(r, a) are the forward and
backward of rank r's segment of it.  The schedule keeps the dependency order
of the pages' scheduling constraints (section 3.1, Eq. 8) restricted to one
layer, where the chunk index is the rank:
    F(r-1, a) < F(r, a)      the state S_in of segment r is S_out of segment r-1
    F(r, a)   < B(r, a)
    B(r+1, a) < B(r, a)      the gradient dS_out of segment r is dS_in of segment r+1
and runs them one-forward-one-backward: rank r does min(M, P - r) forwards
first, then alternates backward and forward, then finishes the backwards.
Sends are non-blocking and receives blocking, which makes the order free of
deadlock; tensors being sent are kept alive until their sends complete.

The arithmetic of a segment is pluggable (``Stage``): ``CudaStage`` runs the
library's sf_gdn_fwd / sf_gdn_bwd on the rank's GPU, keeping only S_in per
microbatch between its forward and backward (the backward recomputes the rest,
as the bounded-memory chain does).  The transport is torch.distributed
point-to-point send/recv (NCCL over NVLink between GPUs).
"""
from __future__ import annotations

import abc
from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Tuple

__all__ = ["schedule", "check_schedule", "Stage", "CudaStage", "SegmentData", "run_pipeline"]


def schedule(P: int, M: int, r: int) -> List[Tuple[str, int]]:
    """Order of rank r's tasks: ("F", a) and ("B", a), one-forward-one-backward."""
    if not (0 <= r < P) or M < 0:
        raise ValueError("need 0 <= r < P and M >= 0")
    out: List[Tuple[str, int]] = []
    nf = nb = 0
    for _ in range(min(M, P - r)):
        out.append(("F", nf))
        nf += 1
    while nb < M:
        out.append(("B", nb))
        nb += 1
        if nf < M:
            out.append(("F", nf))
            nf += 1
    return out


def check_schedule(P: int, M: int) -> int:
    """Simulate all ranks' schedules with the dependency order and blocking
    receives; returns the number of steps the simulation took.  Raises if a
    dependency is violated or the ranks deadlock."""
    order = [schedule(P, M, r) for r in range(P)]
    pos = [0] * P
    done = set()
    steps = 0
    while any(pos[r] < len(order[r]) for r in range(P)):
        progressed = False
        for r in range(P):
            if pos[r] >= len(order[r]):
                continue
            kind, a = order[r][pos[r]]
            if kind == "F":
                ready = r == 0 or ("F", r - 1, a) in done
            else:
                ready = ("F", r, a) in done and (r == P - 1 or ("B", r + 1, a) in done)
            if ready:
                done.add((kind, r, a))
                pos[r] += 1
                progressed = True
        steps += 1
        if not progressed:
            raise RuntimeError(f"pipeline deadlock at step {steps}: {pos}")
    return steps


@dataclass
class SegmentData:
    """Rank r's segment of one microbatch: q, k, v, g, beta, dO of its tokens,
    and for the first rank the sequence's S_in, for the last its dS_out."""
    q: object
    k: object
    v: object
    g: object
    beta: object
    dO: object
    S_in: object = None    # rank 0 only (None = zeros)
    dS_out: object = None  # last rank only (None = zeros)


class Stage(abc.ABC):
    """Arithmetic of one rank's segment.  fwd returns (o, S_out) and keeps what
    bwd needs; bwd returns (grads dict, dS_in); new_state gives an empty fp32
    state tensor [B, H, dk, dv] to receive into."""

    @abc.abstractmethod
    def fwd(self, a: int, seg: SegmentData, S_in):
        ...

    @abc.abstractmethod
    def bwd(self, a: int, seg: SegmentData, dS_out):
        ...

    @abc.abstractmethod
    def new_state(self, seg: SegmentData):
        ...


class CudaStage(Stage):
    """Segment arithmetic on this rank's GPU through the C ABI."""

    def __init__(self, C: int = 64, scale: float = 1.0):
        self.C = C
        self.scale = scale
        self.saved: Dict[int, object] = {}

    def new_state(self, seg):
        import torch
        B, H, _, dk = seg.q.shape
        return torch.empty(B, H, dk, seg.v.shape[-1], dtype=torch.float32, device=seg.q.device)

    def fwd(self, a, seg, S_in):
        from . import fwd
        o, S_out = fwd(seg.q, seg.k, seg.v, seg.g, seg.beta, S_in, C=self.C, scale=self.scale)
        self.saved[a] = S_in
        return o, S_out

    def bwd(self, a, seg, dS_out):
        from . import bwd
        S_in = self.saved.pop(a)
        gr = bwd(seg.q, seg.k, seg.v, seg.g, seg.beta, S_in, seg.dO, dS_out, C=self.C, scale=self.scale)
        return gr, gr["dS_in"]


def run_pipeline(stage: Stage, segments: List[SegmentData], group=None,
                 on_task: Optional[Callable[[str, int], None]] = None):
    """Run the sequence pipeline for this rank over len(segments) microbatches.

    Every rank of ``group`` (default: the world) calls it with its own
    segments, in the same microbatch order.  Returns a list with, per
    microbatch, a dict: o, grads and, on the first rank, dS_in; on the last
    rank, S_out.  ``on_task`` (optional) is called as (kind, a) before each
    task, for tracing."""
    import torch.distributed as dist

    r = dist.get_rank(group)
    P = dist.get_world_size(group)
    M = len(segments)
    to_global = (lambda x: dist.get_global_rank(group, x)) if group is not None else (lambda x: x)
    results: List[dict] = [dict() for _ in range(M)]
    pending = []  # (work, tensor) of sends in flight
    for kind, a in schedule(P, M, r):
        if on_task is not None:
            on_task(kind, a)
        seg = segments[a]
        if kind == "F":
            if r == 0:
                S_in = seg.S_in
            else:
                S_in = stage.new_state(seg)
                dist.recv(S_in, src=to_global(r - 1), group=group)
            o, S_out = stage.fwd(a, seg, S_in)
            results[a]["o"] = o
            if r < P - 1:
                t = S_out.contiguous()
                pending.append((dist.isend(t, dst=to_global(r + 1), group=group), t))
            else:
                results[a]["S_out"] = S_out
        else:
            if r == P - 1:
                dS_out = seg.dS_out
            else:
                dS_out = stage.new_state(seg)
                dist.recv(dS_out, src=to_global(r + 1), group=group)
            grads, dS_in = stage.bwd(a, seg, dS_out)
            results[a]["grads"] = grads
            if r > 0:
                t = dS_in.contiguous()
                pending.append((dist.isend(t, dst=to_global(r - 1), group=group), t))
            else:
                results[a]["dS_in"] = dS_in
    for work, _ in pending:
        work.wait()
    return results
