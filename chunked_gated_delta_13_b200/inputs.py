"""Seeded synthetic inputs for the gated delta-rule layer.

This module only draws random numbers and shapes them into the value
distributions of the workloads (L2-normalised or scaled queries/keys, sigmoid
write strengths, softplus log-decays); it holds none of the layer's arithmetic.
It is the one module that both the CUDA path (tests, benchmark) and the fp64
oracle consume, so both sides see identical values.

Draw order for every workload (CPU ``torch.Generator``, fp32 draws, then a cast):
q, k, v, beta-logits, g-logits, S_in, dO, dS_out.  q, k, v and dO are rounded to
the I/O dtype (bf16 or fp32); g, beta and the states stay fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shape, I/O dtype and value distributions."""
    name: str
    B: int
    H: int
    T: int
    dk: int
    dv: int
    C: int = 64
    io: str = "bf16"                 # "bf16" or "f32"
    use_beta: bool = True
    qk: str = "l2norm"               # "l2norm": N(0,1) then unit L2 norm per token; "scaled": N(0,1)/sqrt(dk)
    g_mode: str = "softplus"         # "softplus": g = -softplus(N(0,1) + g_shift); "zero": g = 0
    g_shift: float = 2.0
    S_in_std: float = 0.0            # 0 -> S_in = 0
    dS_out_std: float = 0.1          # 0 -> dS_out = 0
    N: int = 1                       # segments for the segment chain
    seed: int = 0
    scale: float = 1.0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads of the layer's long-context training settings (Gated
# DeltaNet fwd+bwd at the head counts, head sizes and context lengths of the
# StateFlow evaluation), plus the headline single-GPU shape.
CONFIGS = {
    "c1_f32_small": Workload("c1_f32_small", B=1, H=2, T=256, dk=64, dv=64, C=64, io="f32",
                             S_in_std=0.0, dS_out_std=0.1, N=2),
    "c2_bf16_b2h16": Workload("c2_bf16_b2h16", B=2, H=16, T=8192, dk=128, dv=128, C=64,
                              S_in_std=0.02, dS_out_std=0.1, N=4),
    "c3_chain_h32": Workload("c3_chain_h32", B=1, H=32, T=65536, dk=128, dv=128, C=64,
                             S_in_std=0.0, dS_out_std=0.0, N=16),
    "c4_betaoff_h64": Workload("c4_betaoff_h64", B=1, H=64, T=32768, dk=128, dv=64, C=64,
                               use_beta=False, qk="scaled", g_shift=3.0, S_in_std=0.0,
                               dS_out_std=0.1, N=8),
    "c5_256k": Workload("c5_256k", B=1, H=16, T=262144, dk=128, dv=128, C=64,
                        S_in_std=0.0, dS_out_std=0.0, N=1),
    "headline_h16_t64k": Workload("headline_h16_t64k", B=1, H=16, T=65536, dk=128, dv=128,
                                  C=64, S_in_std=0.0, dS_out_std=0.1, N=1),
    # a small case of the headline shape for profiler captures (inputs still larger than L2)
    "profile_h16_t8k": Workload("profile_h16_t8k", B=1, H=16, T=8192, dk=128, dv=128, C=64,
                                S_in_std=0.0, dS_out_std=0.1, N=1),
}


def _round_io(x: torch.Tensor, io: str) -> torch.Tensor:
    if io == "bf16":
        return x.to(torch.bfloat16)
    if io == "f32":
        return x.to(torch.float32)
    raise ValueError(f"unknown io dtype {io!r}")


def make_inputs(w: Workload) -> dict:
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict of CPU tensors: q, k [B,H,T,dk] and v, dO [B,H,T,dv] in the
    I/O dtype; g, beta [B,H,T] fp32 (beta is None when the beta path is off);
    S_in, dS_out [B,H,dk,dv] fp32 (None when their std is 0).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = randn(B, H, T, dk)
    k = randn(B, H, T, dk)
    if w.qk == "l2norm":
        q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    elif w.qk == "scaled":
        q = q / dk ** 0.5
        k = k / dk ** 0.5
    else:
        raise ValueError(w.qk)
    v = randn(B, H, T, dv)
    beta_logit = randn(B, H, T)
    g_logit = randn(B, H, T)
    beta = torch.sigmoid(beta_logit) if w.use_beta else None
    if w.g_mode == "softplus":
        g = -torch.nn.functional.softplus(g_logit + w.g_shift)
    elif w.g_mode == "zero":
        g = torch.zeros(B, H, T)
    else:
        raise ValueError(w.g_mode)
    S_in = randn(B, H, dk, dv) * w.S_in_std if w.S_in_std > 0 else None
    dO = randn(B, H, T, dv)
    dS_out = randn(B, H, dk, dv) * w.dS_out_std if w.dS_out_std > 0 else None
    return {
        "q": _round_io(q, w.io), "k": _round_io(k, w.io), "v": _round_io(v, w.io),
        "g": g.contiguous(), "beta": None if beta is None else beta.contiguous(),
        "S_in": S_in, "dO": _round_io(dO, w.io), "dS_out": dS_out,
    }


def as_f64(inputs: dict) -> dict:
    """The same values upcast to numpy fp64 (what the oracle consumes)."""
    out = {}
    for name, t in inputs.items():
        out[name] = None if t is None else t.to(torch.float64).numpy()
    return out


@dataclass(frozen=True)
class ConvWorkload:
    """Synthetic inputs of the short causal convolution: x ~ N(0,1), taps
    w ~ N(0, 1/K), boundary state ~ N(0,1) (or none), dy ~ N(0,1), boundary-state
    gradient ~ N(0, 0.1) (or none)."""
    name: str
    B: int
    H: int
    T: int
    d: int
    K: int = 4
    io: str = "bf16"
    act: str = "silu"
    with_state: bool = True
    seed: int = 0

    def with_(self, **kw) -> "ConvWorkload":
        return replace(self, **kw)


def make_conv_inputs(w: ConvWorkload) -> dict:
    """Draw order: x, taps, conv_in, dy, dconv_out (CPU generator, fp32 draws)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    x = randn(w.B, w.H, w.T, w.d)
    taps = randn(w.H, w.d, w.K) / w.K ** 0.5
    ci = randn(w.B, w.H, w.K - 1, w.d)
    dy = randn(w.B, w.H, w.T, w.d)
    dco = randn(w.B, w.H, w.K - 1, w.d) * 0.1
    return {"x": _round_io(x, w.io), "w": taps.contiguous(),
            "conv_in": _round_io(ci, w.io) if w.with_state else None,
            "dy": _round_io(dy, w.io), "dconv_out": dco if w.with_state else None}


def make_kda_inputs(w: Workload) -> dict:
    """Inputs of the per-channel-decay variant: as make_inputs, with the
    log-decay drawn per key channel, g = -softplus(N(0,1) + g_shift) of shape
    [B,H,T,dk] (g_mode "zero": all zeros).  Draw order: q, k, v, beta-logits,
    g-logits, S_in, dO, dS_out."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed)
    B, H, T, dk, dv = w.B, w.H, w.T, w.dk, w.dv

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = randn(B, H, T, dk)
    k = randn(B, H, T, dk)
    if w.qk == "l2norm":
        q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-12)
    else:
        q = q / dk ** 0.5
        k = k / dk ** 0.5
    v = randn(B, H, T, dv)
    beta_logit = randn(B, H, T)
    g_logit = randn(B, H, T, dk)
    beta = torch.sigmoid(beta_logit) if w.use_beta else None
    g = (-torch.nn.functional.softplus(g_logit + w.g_shift) if w.g_mode == "softplus"
         else torch.zeros(B, H, T, dk))
    S_in = randn(B, H, dk, dv) * w.S_in_std if w.S_in_std > 0 else None
    dO = randn(B, H, T, dv)
    dS_out = randn(B, H, dk, dv) * w.dS_out_std if w.dS_out_std > 0 else None
    return {"q": _round_io(q, w.io), "k": _round_io(k, w.io), "v": _round_io(v, w.io),
            "g": g.contiguous(), "beta": None if beta is None else beta.contiguous(),
            "S_in": S_in, "dO": _round_io(dO, w.io), "dS_out": dS_out}
