"""GPU parity of gdn_chunk_fwd_host (host buffers, the sequence pipelined through
the device piece by piece) against the fp64 oracle, and its agreement with the
device entry point (max|err|/RMS per tensor, raw: 1e-4 for float32 inputs, 2e-2 for
bf16 inputs, on float32 outputs; the bf16 output is checked to be their rounding)."""
import pytest
import torch

from gdn_synth import gdn_inputs
from oracle import oracle as O
from tests.parity import TOL, assert_bf16_store, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _host(x):
    return {n: (t.cpu().pin_memory() if t is not None else None) for n, t in x.items()}


CASES = [  # B, T, Hk, Hv, d, dtype, piece_tokens
    (1, 300, 2, 4, 128, torch.bfloat16, 128),   # three pieces, ragged last piece
    (2, 257, 1, 2, 128, torch.bfloat16, 64),    # five pieces of one chunk, two batch rows
    (1, 1000, 2, 8, 128, torch.bfloat16, 0),    # default piece size
    (2, 130, 2, 4, 64, torch.float32, 64),      # float32 CUDA-core path, three pieces
    (1, 40, 1, 1, 128, torch.bfloat16, 512),    # one piece shorter than a chunk
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:5]) + str(c[6]) for c in CASES])
def test_host_pipeline_matches_oracle(case):
    B, T, Hk, Hv, d, dtype, piece = case
    x = gdn_inputs(B, T, Hk, Hv, d, dtype, seed=700 + T, device=DEV)
    h = _host(x)
    o, ht = G.gdn_chunk_fwd_host(h["q"], h["k"], h["v"], h["a"], h["b"], h["A_log"],
                                 h["dt_bias"], h["h0"], piece_tokens=piece, out_f32=True)
    torch.cuda.synchronize()
    assert not o.is_cuda and not ht.is_cuda
    if dtype == torch.bfloat16:
        o16, ht16 = G.gdn_chunk_fwd_host(h["q"], h["k"], h["v"], h["a"], h["b"], h["A_log"],
                                         h["dt_bias"], h["h0"], piece_tokens=piece)
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    tol = TOL[dtype]
    assert rel_err(o, ro) <= tol
    assert rel_err(ht, rht) <= tol
    # the same result as the device entry point on the same inputs
    od, htd = G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                              x["h0"], out_f32=True)
    assert rel_err(o, od.cpu().double()) <= tol
    assert rel_err(ht, htd.cpu().double()) <= tol


def test_host_pipeline_zero_state_and_precomputed_gates():
    """GDN_GATES_PRECOMPUTED with the oracle's own g, beta, and no initial state."""
    B, T, Hk, Hv, d = 1, 200, 2, 4, 128
    x = gdn_inputs(B, T, Hk, Hv, d, torch.bfloat16, seed=811, device=DEV)
    _, _, g, beta = O.gate_prep(cpu(x["q"]), cpu(x["k"]), cpu(x["a"]), cpu(x["b"]),
                                cpu(x["A_log"]), cpu(x["dt_bias"]))
    g32 = torch.from_numpy(g).float().pin_memory()
    b32 = torch.from_numpy(beta).float().pin_memory()
    h = _host(x)
    o, ht = G.gdn_chunk_fwd_host(h["q"], h["k"], h["v"], g32, b32, None, None, None,
                                 gates_precomputed=True, piece_tokens=64, out_f32=True)
    torch.cuda.synchronize()
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(g32), cpu(b32), h0=None,
                        gates_given=True)
    assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2


def test_host_pipeline_workspace_checks():
    x = _host(gdn_inputs(1, 128, 1, 1, 128, torch.bfloat16, seed=5, device=DEV))
    need = G.gdn_chunk_fwd_host_workspace_bytes(1, 128, 1, 1, 128, 128, torch.bfloat16,
                                                piece_tokens=64)
    assert need > 0
    small = torch.empty(need - 256, device=DEV, dtype=torch.uint8)
    with pytest.raises(G.GDNError) as e:
        G.gdn_chunk_fwd_host(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                             x["h0"], piece_tokens=64, dev_workspace=small)
    assert e.value.status == -5  # GDN_ERR_WORKSPACE
