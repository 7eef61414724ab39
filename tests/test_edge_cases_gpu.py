"""GPU parity on the method's degenerate cases, through GDN_GATES_PRECOMPUTED, on
both tensor-core paths (GDN and Gated DeltaNet-2, bf16, d = 128) and the float32
CUDA-core path, each against the fp64 oracle on the same inputs, over several
chunks with a ragged tail:

  overwrite       g = 0, beta = 1 on orthonormal keys, keys rewritten inside a
                  chunk and across chunks ("从 Full Attention 到 Gated DeltaNet" §6:
                  the delta rule replaces the value stored under a key);
  pure decay      beta = 0 (no erase, no write): S_t = (prod alpha) S_0;
  linear attn.    Gated DeltaNet-2 with D = I, b = 0, w = 1: S_t = S_{t-1} + k v^T
                  ("Gated DeltaNet-2", 退化兼容性);
  saturated decay g = -50 per token (alpha ~ 2e-22): only the newest token survives.

They stress the per-CTA range scale of the scan and the log-domain gate factors
at their extremes.  Also: values of magnitude ~1e6 stay within the bar (the range
scale absorbs them), and queries / keys of norm ~1e4 with the norm off report
GDN_ERR_RANGE instead of returning silently wrong outputs.
"""
import numpy as np
import pytest
import torch

from gdn_synth import gdn2_inputs, gdn_inputs
from oracle import oracle as O
from tests.parity import TOL, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"
D = 128


def _orthonormal_keys(T, period, seed, dtype):
    """Key t is row (t mod period) of a random orthogonal matrix: every key is
    rewritten every `period` tokens (inside a chunk when period < 64)."""
    g = torch.Generator().manual_seed(seed)
    Qm, _ = torch.linalg.qr(torch.randn(D, D, generator=g, dtype=torch.float64))
    idx = torch.arange(T) % period
    return Qm[idx].to(dtype)  # [T, D]


def _gdn_case(case, T, dtype, seed):
    """q, k [1,T,Hk,D], v [1,T,Hv,D], g, beta [1,T,Hv] float32, h0, for Hk=1, Hv=2."""
    Hk, Hv = 1, 2
    x = gdn_inputs(1, T, Hk, Hv, D, dtype, seed=seed, device="cpu")
    gen = torch.Generator().manual_seed(seed + 1)
    q, k, v, h0 = x["q"], x["k"], x["v"], x["h0"]
    g = torch.zeros(1, T, Hv)
    beta = torch.full((1, T, Hv), 1.0)
    if case == "overwrite":
        keys = _orthonormal_keys(T, 48, seed, dtype)
        k = keys.view(1, T, 1, D).contiguous()
        q = _orthonormal_keys(T, 40, seed, dtype).view(1, T, 1, D).contiguous()
    elif case == "pure_decay":
        beta.zero_()
        g = -0.02 * torch.rand(1, T, Hv, generator=gen)
        h0 = torch.randn(1, Hv, D, D, generator=gen)
        q = torch.nn.functional.normalize(q.float(), dim=-1).to(dtype)
    elif case == "saturated":
        g = torch.full((1, T, Hv), -50.0)
        beta = torch.sigmoid(torch.randn(1, T, Hv, generator=gen))
        q = torch.nn.functional.normalize(q.float(), dim=-1).to(dtype)
        k = torch.nn.functional.normalize(k.float(), dim=-1).to(dtype)
    else:
        raise ValueError(case)
    return q, k, v, g.float(), beta.float(), h0


def _gdn2_case(case, T, dtype, seed):
    H = 2
    x = gdn2_inputs(1, T, H, D, dtype, seed=seed, device="cpu")
    gen = torch.Generator().manual_seed(seed + 1)
    q, k, v, h0 = x["q"], x["k"], x["v"], x["h0"]
    q = torch.nn.functional.normalize(q.float(), dim=-1).to(dtype)
    k = torch.nn.functional.normalize(k.float(), dim=-1).to(dtype)
    g = torch.zeros(1, T, H, D)
    bg = torch.ones(1, T, H, D)
    wg = torch.ones(1, T, H, D)
    if case == "overwrite":
        k = _orthonormal_keys(T, 48, seed, dtype).view(1, T, 1, D).expand(1, T, H, D).contiguous()
        q = _orthonormal_keys(T, 40, seed, dtype).view(1, T, 1, D).expand(1, T, H, D).contiguous()
    elif case == "pure_decay":
        bg.zero_()
        wg.zero_()
        g = -0.02 * torch.rand(1, T, H, D, generator=gen)
        h0 = torch.randn(1, H, D, D, generator=gen)
    elif case == "linear_attention":
        bg.zero_()
    elif case == "saturated":
        g = torch.full((1, T, H, D), -50.0)
        bg = torch.sigmoid(torch.randn(1, T, H, D, generator=gen))
        wg = torch.sigmoid(torch.randn(1, T, H, D, generator=gen))
    else:
        raise ValueError(case)
    return q, k, v, g.float(), bg.float(), wg.float(), h0


def _dev(*ts):
    return [None if t is None else t.to(DEV) for t in ts]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [256, 300])
@pytest.mark.parametrize("case", ["overwrite", "pure_decay", "saturated"])
def test_gdn_degenerate_cases(case, T, dtype):
    q, k, v, g, beta, h0 = _gdn_case(case, T, dtype, seed=900 + T)
    scale = 1.0
    dq, dk_, dv, dg, db, dh0 = _dev(q, k, v, g, beta, h0)
    o, ht = G.gdn_chunk_fwd(dq, dk_, dv, dg, db, None, None, dh0, l2norm=False,
                            gates_precomputed=True, scale=scale, out_f32=True)
    assert G.gdn_status() == 0
    ro, rht = O.gdn_fwd(q, k, v, g, beta, h0=h0, scale=scale, l2norm=False, gates_given=True)
    eo, eh = rel_err(o, ro), rel_err(ht, rht)
    assert eo <= TOL[dtype] and eh <= TOL[dtype], (eo, eh)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [256, 300])
@pytest.mark.parametrize("case", ["overwrite", "pure_decay", "linear_attention", "saturated"])
def test_gdn2_degenerate_cases(case, T, dtype):
    q, k, v, g, bg, wg, h0 = _gdn2_case(case, T, dtype, seed=950 + T)
    scale = 1.0
    dq, dk_, dv, dg, dbg, dwg, dh0 = _dev(q, k, v, g, bg, wg, h0)
    o, ht = G.gdn2_chunk_fwd(dq, dk_, dv, dg, dbg, dwg, None, None, dh0, scale=scale,
                             l2norm=False, gates_precomputed=True, out_f32=True)
    assert G.gdn_status() == 0
    ro, rht = O.gdn2_fwd(q, k, v, g, bg, wg, h0=h0, scale=scale, l2norm=False,
                         gates_given=True)
    eo, eh = rel_err(o, ro), rel_err(ht, rht)
    assert eo <= TOL[dtype] and eh <= TOL[dtype], (eo, eh)


def test_overwrite_retrieves_the_newest_value():
    """On the overwrite case the oracle itself returns, for a query equal to a
    stored key, the value written last under it (alpha = beta = 1, orthonormal
    keys, zero initial state); the GPU output matches that retrieval."""
    T = 256
    keys = _orthonormal_keys(T, 48, 5, torch.bfloat16)
    k = keys.view(1, T, 1, D).contiguous()
    q = k.clone()
    v = torch.randn(1, T, 1, D, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    g = torch.zeros(1, T, 1)
    beta = torch.ones(1, T, 1)
    o, _ = G.gdn_chunk_fwd(*_dev(q, k, v, g, beta), None, None, None, l2norm=False,
                           gates_precomputed=True, scale=1.0, out_f32=True)
    ro, _ = O.gdn_fwd(q, k, v, g, beta, h0=None, scale=1.0, l2norm=False, gates_given=True)
    # query t = key t was written at token t: the retrieval is v_t up to the bf16
    # rounding of the keys (not exactly orthonormal after rounding)
    vt = v[0, :, 0].double().numpy()
    assert np.max(np.abs(ro[0, :, 0] - vt)) / np.sqrt(np.mean(vt ** 2)) < 5e-2
    assert rel_err(o, ro) <= 2e-2


def test_large_values_are_absorbed_by_the_range_scale():
    """v ~ N(0, 1e12): the scan's power-of-2 range scale keeps every fp16 operand in
    range; parity holds and no range error is reported."""
    x = gdn_inputs(1, 200, 1, 2, D, torch.bfloat16, seed=31, device="cpu")
    x["v"] = (x["v"].float() * 1e6).to(torch.bfloat16)
    x["h0"] = x["h0"] * 1e6
    d = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    o, ht = G.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                            d["h0"], out_f32=True)
    assert G.gdn_status() == 0
    ro, rht = O.gdn_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"])
    assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2


def test_out_of_range_operands_report_range_error():
    """Queries and keys of norm ~1e4 with the L2 norm off put A_qk = q.k far past the
    fp16 range: the call reports GDN_ERR_RANGE (its outputs are not to be used)."""
    x = gdn_inputs(1, 130, 1, 2, D, torch.bfloat16, seed=32, device=DEV)
    q = (x["q"].float() * 1e3).to(torch.bfloat16)
    k = (x["k"].float() * 1e3).to(torch.bfloat16)
    G.gdn_chunk_fwd(q, k, x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"], x["h0"],
                    l2norm=False)
    assert G.gdn_status() == -6  # GDN_ERR_RANGE (read and cleared)
    # the status word is clean again and an in-range call is green
    o, ht = G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                            x["h0"])
    assert G.gdn_status() == 0
