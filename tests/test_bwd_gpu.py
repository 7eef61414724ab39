"""GPU parity of the chunk backward (gdn_chunk_bwd) against the oracle's token-by-
token reverse-mode backward (oracle.gdn_bwd), on the same seeded inputs and output
gradients: every gradient (dq, dk, dv, da, db, dA_log, ddt_bias, dh0) element by
element, bar max |err| / RMS(ref) <= 1e-4 for float32 inputs and <= 2e-2 for bf16
inputs (the backward computes in float32 for both; its float32 outputs are held to
the bar raw).  Cases span several chunks with ragged tails, GQA groups, d = 64 and
128, the norm on and off, gates from logits and given directly, with and without
the initial state and the final-state gradient; plus T = 0, the workspace check,
and the prefill_8k layer at full size on the heads of one key-head group."""
import numpy as np
import pytest
import torch

from gdn_synth import WORKLOADS, bwd_cotangents, gdn_inputs, workload_inputs
from oracle import oracle as O
from tests.parity import TOL, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"
NAMES = ("dq", "dk", "dv", "da", "db", "dA_log", "ddt_bias", "dh0")


def _check(got, ref, tol, heads=None):
    for n in NAMES:
        if ref[n] is None or got[n] is None:
            continue
        g = got[n]
        if heads is not None:  # a sample of heads: (key-head slice, value-head slice)
            hk, hv = heads
            g = {"dq": lambda t: t[:, :, hk], "dk": lambda t: t[:, :, hk],
                 "dv": lambda t: t[:, :, hv], "da": lambda t: t[:, :, hv],
                 "db": lambda t: t[:, :, hv], "dA_log": lambda t: t[hv],
                 "ddt_bias": lambda t: t[hv], "dh0": lambda t: t[:, hv]}[n](g)
        err = rel_err(g, ref[n])
        assert err <= tol, f"{n}: {err:.3e} > {tol}"


def _gates_given(x):
    _, _, g, beta = O.gate_prep(cpu(x["q"]), cpu(x["k"]), cpu(x["a"]), cpu(x["b"]),
                                cpu(x["A_log"]), cpu(x["dt_bias"]))
    return (torch.from_numpy(g).float().to(DEV), torch.from_numpy(beta).float().to(DEV))


CASES = [
    # B, T, Hk, Hv, d, dtype, l2norm, gates given, h0, dht
    (1, 1, 1, 1, 64, torch.float32, True, False, False, False),
    (1, 63, 1, 2, 64, torch.float32, True, False, True, True),
    (1, 64, 2, 2, 128, torch.bfloat16, True, False, False, True),
    (2, 65, 1, 4, 128, torch.bfloat16, True, False, True, True),
    (1, 130, 2, 4, 64, torch.float32, True, True, True, False),
    (1, 200, 1, 2, 128, torch.float32, False, True, False, True),
    (2, 300, 2, 8, 128, torch.bfloat16, True, False, True, True),
    (1, 190, 1, 1, 128, torch.float32, True, False, True, True),
]


@pytest.mark.parametrize("B,T,Hk,Hv,d,dtype,l2,pre,h0,dht", CASES)
def test_chunk_bwd_matches_oracle(B, T, Hk, Hv, d, dtype, l2, pre, h0, dht):
    x = gdn_inputs(B, T, Hk, Hv, d, dtype, seed=300 + T + d, device=DEV, h0=h0)
    ct = bwd_cotangents(B, T, Hv, d, d, dtype, seed=400 + T, device=DEV, dht=dht)
    a, b = _gates_given(x) if pre else (x["a"], x["b"])
    q, k = x["q"], x["k"]
    if pre and not l2:  # unit-norm keys with the norm off, as the method expects
        q = torch.nn.functional.normalize(q.float(), dim=-1).to(dtype)
        k = torch.nn.functional.normalize(k.float(), dim=-1).to(dtype)
    scale = d ** -0.5
    got = G.gdn_chunk_bwd(q, k, x["v"], a, b, x["A_log"], x["dt_bias"], x["h0"], ct["do"],
                          ct["dht"], scale=scale, l2norm=l2, gates_precomputed=pre)
    torch.cuda.synchronize()
    ref = O.gdn_bwd(cpu(q), cpu(k), cpu(x["v"]), cpu(a), cpu(b), cpu(x["A_log"]),
                    cpu(x["dt_bias"]), cpu(x["h0"]), cpu(ct["do"]), cpu(ct["dht"]), scale=scale,
                    l2norm=l2, gates_given=pre)
    _check(got, ref, TOL[dtype])


def test_chunk_bwd_empty_sequence():
    """T = 0: dh0 equals dht and the gate parameters get zero gradient."""
    x = gdn_inputs(2, 0, 1, 2, 64, torch.float32, seed=5, device=DEV)
    ct = bwd_cotangents(2, 0, 2, 64, 64, torch.float32, seed=6, device=DEV)
    got = G.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                          x["h0"], ct["do"], ct["dht"])
    torch.cuda.synchronize()
    assert torch.equal(got["dh0"], ct["dht"])
    assert torch.count_nonzero(got["dA_log"]) == 0 and torch.count_nonzero(got["ddt_bias"]) == 0


def test_chunk_bwd_workspace_checked():
    x = gdn_inputs(1, 100, 1, 2, 64, torch.float32, seed=7, device=DEV)
    ct = bwd_cotangents(1, 100, 2, 64, 64, torch.float32, seed=8, device=DEV)
    need = G.gdn_chunk_bwd_workspace_bytes(1, 100, 1, 2, 64, 64)
    assert need > 0
    small = torch.empty(need - 256, device=DEV, dtype=torch.uint8)
    with pytest.raises(G.GDNError):
        G.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                        x["h0"], ct["do"], workspace=small)


def test_chunk_bwd_prefill_8k_full_size_sampled_heads():
    """The prefill_8k layer (B=1, T=8192, 16 key heads, 64 value heads, d=128, bf16) in
    one backward call; the oracle recomputes key head 0 and its four value heads."""
    w = WORKLOADS["prefill_8k"]
    x = workload_inputs(w, DEV)
    ct = bwd_cotangents(w.B, w.T, w.Hv, w.d, w.d, w.dtype, seed=1501, device=DEV)
    got = G.gdn_chunk_bwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                          x["h0"], ct["do"], ct["dht"])
    torch.cuda.synchronize()
    Gq = w.Hv // w.Hk
    hv = slice(0, Gq)
    ref = O.gdn_bwd(cpu(x["q"][:, :, 0:1]), cpu(x["k"][:, :, 0:1]), cpu(x["v"][:, :, hv]),
                    cpu(x["a"][:, :, hv]), cpu(x["b"][:, :, hv]), cpu(x["A_log"][hv]),
                    cpu(x["dt_bias"][hv]), cpu(x["h0"][:, hv]), cpu(ct["do"][:, :, hv]),
                    cpu(ct["dht"][:, hv]), scale=w.d ** -0.5)
    _check(got, ref, TOL[w.dtype], heads=(slice(0, 1), hv))
