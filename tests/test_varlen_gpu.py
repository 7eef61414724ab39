"""GPU parity of gdn_chunk_fwd_varlen: a packed batch of sequences of different
lengths (empty and single-token ones included), each against the oracle on its
own tokens and state, and bit for bit against one-sequence gdn_chunk_fwd calls."""
import pytest
import torch

from gdn_synth import gdn_inputs
from oracle import oracle as O
from tests.parity import TOL, assert_bf16_store, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_varlen_packed_batch(dtype, d):
    lens = [5, 64, 0, 130, 1]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    N, Tt, Hk, Hv = len(lens), cu[-1], 2, 4
    x = gdn_inputs(1, Tt, Hk, Hv, d, dtype, seed=90, device=DEV, h0=False)
    h0 = 0.02 * torch.randn(N, Hv, d, d, device=DEV)
    q, k, v, a, b = (x[n][0] for n in ("q", "k", "v", "a", "b"))
    o, ht = G.gdn_chunk_fwd_varlen(q, k, v, a, b, x["A_log"], x["dt_bias"], h0, cu,
                                   out_f32=True)
    if dtype == torch.bfloat16:
        o16, ht16 = G.gdn_chunk_fwd_varlen(q, k, v, a, b, x["A_log"], x["dt_bias"], h0, cu)
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)
    tol = TOL[dtype]
    for i in range(N):
        s0, s1 = cu[i], cu[i + 1]
        sl = lambda t: t[s0:s1][None]
        o1, h1 = G.gdn_chunk_fwd(sl(q), sl(k), sl(v), sl(a), sl(b), x["A_log"], x["dt_bias"],
                                 h0[i:i + 1], out_f32=True)
        assert torch.equal(o[s0:s1], o1[0]) and torch.equal(ht[i], h1[0])
        ro, rht = O.gdn_fwd(cpu(sl(q)), cpu(sl(k)), cpu(sl(v)), cpu(sl(a)), cpu(sl(b)),
                            cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(h0[i:i + 1]))
        if s1 > s0:
            assert rel_err(o[s0:s1], ro[0]) <= tol
        assert rel_err(ht[i], rht[0]) <= tol
