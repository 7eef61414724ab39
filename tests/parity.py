"""Shared helpers of the GPU parity tests: the error metric and tolerances.

Metric (per output tensor): max |gpu - oracle| / RMS(oracle); bars 1e-4 for
float32 inputs and 2e-2 for bf16 inputs (float32 accumulation and state).

Outputs stored in bf16 carry, on top of the computation's own error, the
rounding of the final store: |rn(o) - o| <= u |o| with u = 2^-8 (bf16 keeps
8 significant bits).  Since |o_bf16 - ref| <= |o - ref| + u (|ref| + |o - ref|),
the error of the computation before that store is at least
(|o_bf16 - ref| - u |ref|) / (1 + u) per element; that is the per-element
error the bar is applied to for bf16 outputs.  Outputs written in float32
(GDN_OUT_F32) get no allowance.  conv_state is a byte copy and is compared bit
for bit.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
U_BF16 = 2.0 ** -8


def rel_err(x, ref) -> float:
    bf16_out = hasattr(x, "dtype") and x.dtype == torch.bfloat16
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().double().numpy()
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in the GPU result"
    err = np.abs(x - ref)
    if bf16_out:
        err = np.maximum(err - U_BF16 * np.abs(ref), 0.0) / (1.0 + U_BF16)
    rms = float(np.sqrt(np.mean(ref * ref)))
    if rms == 0.0:
        return float(np.max(err)) if err.size else 0.0
    return float(np.max(err) / rms) if err.size else 0.0


def cpu(t):
    return None if t is None else t.detach().cpu()
