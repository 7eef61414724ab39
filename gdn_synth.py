"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module only draws random numbers with fixed seeds, shapes and
distributions; it holds none of the method's arithmetic.  The CUDA library and
the oracle both consume the tensors it returns (the oracle after a plain copy
to the host), so both sides see bit-identical input values.

Shapes follow the Qwen3.5 GDN layer the pages describe (16 key heads, 64 value
heads, head dim 128, causal conv kernel 4, contexts up to 256K); distributions
follow the workload list of the build: q, k, v, a, b ~ N(0,1); A_log ~ U(0, ln 16);
dt_bias ~ U(-4, -1); initial state ~ N(0, 0.02^2) in fp32; conv weights
~ U(-0.5, 0.5); conv state ~ N(0, 1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

LN16 = math.log(16.0)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "gdn" | "decode" | "gdn2" | "conv" | "norm"
    B: int
    T: int
    Hk: int
    Hv: int
    d: int
    dtype: torch.dtype
    seed: int
    h0: bool = True
    steps: int = 1       # decode only: consecutive steps
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.B * self.T if self.kind != "decode" else self.B * self.steps


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", "gdn", 1, 256, 2, 2, 64, torch.float32, 1000, h0=False),
    "prefill_8k": Workload("prefill_8k", "gdn", 1, 8192, 16, 64, 128, torch.bfloat16, 1001),
    "prefill_128k": Workload("prefill_128k", "gdn", 1, 131072, 16, 64, 128, torch.bfloat16, 1002),
    "prefill_b8_16k": Workload("prefill_b8_16k", "gdn", 8, 16384, 16, 64, 128, torch.bfloat16, 1002),
    "decode_256": Workload("decode_256", "decode", 256, 1, 16, 64, 128, torch.bfloat16, 1003, steps=64),
    "gdn2_b4_4k": Workload("gdn2_b4_4k", "gdn2", 4, 4096, 16, 16, 128, torch.bfloat16, 1004),
    # the prefill conv1d + SiLU over the mixed stream of the prefill_8k layer
    "conv_prefill_8k": Workload("conv_prefill_8k", "conv", 1, 8192, 16, 64, 128, torch.bfloat16,
                                1005),
    # the gated RMSNorm of the prefill_8k layer's core output
    "rmsnorm_gated_8k": Workload("rmsnorm_gated_8k", "norm", 1, 8192, 16, 64, 128,
                                 torch.bfloat16, 1006),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, gen, device, dtype, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _uniform(shape, lo, hi, gen, device):
    return torch.rand(shape, generator=gen, device=device, dtype=torch.float32) * (hi - lo) + lo


def gdn_inputs(B, T, Hk, Hv, d, dtype, seed, device="cpu", h0=True, dv=None):
    """Inputs of one GDN prefill call.

    q, k [B,T,Hk,d]; v [B,T,Hv,dv]; a, b [B,T,Hv] in ``dtype``;
    A_log, dt_bias [Hv] fp32; h0 [B,Hv,d,dv] fp32 (or None).
    """
    dv = d if dv is None else dv
    g = _gen(seed, device)
    out = {
        "q": _randn((B, T, Hk, d), g, device, dtype),
        "k": _randn((B, T, Hk, d), g, device, dtype),
        "v": _randn((B, T, Hv, dv), g, device, dtype),
        "a": _randn((B, T, Hv), g, device, dtype),
        "b": _randn((B, T, Hv), g, device, dtype),
        "A_log": _uniform((Hv,), 0.0, LN16, g, device),
        "dt_bias": _uniform((Hv,), -4.0, -1.0, g, device),
    }
    out["h0"] = _randn((B, Hv, d, dv), g, device, torch.float32, std=0.02) if h0 else None
    return out


def gdn2_inputs(B, T, H, d, dtype, seed, device="cpu", h0=True, dv=None):
    """Inputs of one Gated DeltaNet-2 call.

    q, k [B,T,H,d]; v [B,T,H,dv]; a, b_logit [B,T,H,d]; w_logit [B,T,H,dv];
    A_log, dt_bias [H,d] fp32; h0 [B,H,d,dv] fp32 (or None).
    """
    dv = d if dv is None else dv
    g = _gen(seed, device)
    out = {
        "q": _randn((B, T, H, d), g, device, dtype),
        "k": _randn((B, T, H, d), g, device, dtype),
        "v": _randn((B, T, H, dv), g, device, dtype),
        "a": _randn((B, T, H, d), g, device, dtype),
        "b_logit": _randn((B, T, H, d), g, device, dtype),
        "w_logit": _randn((B, T, H, dv), g, device, dtype),
        "A_log": _uniform((H, d), 0.0, LN16, g, device),
        "dt_bias": _uniform((H, d), -4.0, -1.0, g, device),
    }
    out["h0"] = _randn((B, H, d, dv), g, device, torch.float32, std=0.02) if h0 else None
    return out


def decode_inputs(N, steps, Hk, Hv, d, dtype, seed, device="cpu", dv=None):
    """Inputs of `steps` consecutive decode steps for N sequences.

    x [steps,N,Cc] pre-conv mixed [q|k|v] stream, Cc = 2*Hk*d + Hv*dv;
    conv_w [Cc,4] fp32; conv_state [N,Cc,3] ``dtype``; a, b [steps,N,Hv];
    A_log, dt_bias [Hv] fp32; state [N,Hv,d,dv] fp32.
    """
    dv = d if dv is None else dv
    Cc = 2 * Hk * d + Hv * dv
    g = _gen(seed, device)
    return {
        "x": _randn((steps, N, Cc), g, device, dtype),
        "conv_w": _uniform((Cc, 4), -0.5, 0.5, g, device),
        "conv_state": _randn((N, Cc, 3), g, device, dtype),
        "a": _randn((steps, N, Hv), g, device, dtype),
        "b": _randn((steps, N, Hv), g, device, dtype),
        "A_log": _uniform((Hv,), 0.0, LN16, g, device),
        "dt_bias": _uniform((Hv,), -4.0, -1.0, g, device),
        "state": _randn((N, Hv, d, dv), g, device, torch.float32, std=0.02),
    }


def conv_prefill_inputs(B, T, Hk, Hv, d, dtype, seed, device="cpu", dv=None):
    """Inputs of one prefill conv call: x [B,T,Cc] pre-conv mixed [q|k|v] stream,
    Cc = 2*Hk*d + Hv*dv, in ``dtype``; conv_w [Cc,4] fp32; conv_state [B,Cc,3]
    ``dtype`` (the same distributions as the decode inputs)."""
    dv = d if dv is None else dv
    Cc = 2 * Hk * d + Hv * dv
    g = _gen(seed, device)
    return {
        "x": _randn((B, T, Cc), g, device, dtype),
        "conv_w": _uniform((Cc, 4), -0.5, 0.5, g, device),
        "conv_state": _randn((B, Cc, 3), g, device, dtype),
    }


def kda_inputs(B, T, H, d, dtype, seed, device="cpu", h0=True, dv=None):
    """Inputs of one KDA call: q, k [B,T,H,d]; v [B,T,H,dv]; a [B,T,H,d] (per-channel
    decay input) and beta [B,T,H] (logit) in ``dtype``; A_log, dt_bias [H,d] fp32 as
    for Gated DeltaNet-2; h0 [B,H,d,dv] fp32 (or None)."""
    dv = d if dv is None else dv
    g = _gen(seed, device)
    out = {
        "q": _randn((B, T, H, d), g, device, dtype),
        "k": _randn((B, T, H, d), g, device, dtype),
        "v": _randn((B, T, H, dv), g, device, dtype),
        "a": _randn((B, T, H, d), g, device, dtype),
        "beta": _randn((B, T, H), g, device, dtype),
        "A_log": _uniform((H, d), 0.0, LN16, g, device),
        "dt_bias": _uniform((H, d), -4.0, -1.0, g, device),
    }
    out["h0"] = _randn((B, H, d, dv), g, device, torch.float32, std=0.02) if h0 else None
    return out


def rmsnorm_inputs(B, T, Hv, dv, dtype, seed, device="cpu"):
    """Inputs of one gated RMSNorm call: the core output o and the gate z
    [B,T,Hv,dv] ~ N(0,1) in ``dtype``; weight [dv] ~ U(0.5, 1.5) fp32."""
    g = _gen(seed, device)
    return {
        "o": _randn((B, T, Hv, dv), g, device, dtype),
        "z": _randn((B, T, Hv, dv), g, device, dtype),
        "weight": _uniform((dv,), 0.5, 1.5, g, device),
    }


def bwd_cotangents(B, T, Hv, dv, dk, dtype, seed, device="cpu", dht=True):
    """Gradients at the outputs of one GDN call, for its backward: do [B,T,Hv,dv]
    ~ N(0,1) in ``dtype``; dht [B,Hv,dk,dv] ~ N(0,1) fp32 (or None)."""
    g = _gen(seed, device)
    return {"do": _randn((B, T, Hv, dv), g, device, dtype),
            "dht": _randn((B, Hv, dk, dv), g, device, torch.float32) if dht else None}


def workload_inputs(w: Workload, device="cpu"):
    if w.kind == "gdn":
        return gdn_inputs(w.B, w.T, w.Hk, w.Hv, w.d, w.dtype, w.seed, device, h0=w.h0)
    if w.kind == "gdn2":
        return gdn2_inputs(w.B, w.T, w.Hv, w.d, w.dtype, w.seed, device, h0=w.h0)
    if w.kind == "decode":
        return decode_inputs(w.B, w.steps, w.Hk, w.Hv, w.d, w.dtype, w.seed, device)
    if w.kind == "conv":
        return conv_prefill_inputs(w.B, w.T, w.Hk, w.Hv, w.d, w.dtype, w.seed, device)
    if w.kind == "norm":
        return rmsnorm_inputs(w.B, w.T, w.Hv, w.d, w.dtype, w.seed, device)
    raise ValueError(w.kind)
