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


def _packed(lens, Hk, Hv, d, dtype, seed):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    x = gdn_inputs(1, cu[-1], Hk, Hv, d, dtype, seed=seed, device=DEV, h0=False)
    h0 = 0.02 * torch.randn(len(lens), Hv, d, d, device=DEV)
    return cu, x, h0, [x[n][0] for n in ("q", "k", "v", "a", "b")]


def test_varlen_many_mixed_lengths_in_one_launch_pair():
    """64 sequences of mixed length (empty, single-token, chunk-aligned, ragged, a
    few chunks) through the packed launch pair: bit for bit the one-sequence
    calls, and the oracle on a sample of them."""
    g = torch.Generator().manual_seed(7)
    pool = [0, 1, 2, 63, 64, 65, 127, 128, 129, 200, 300, 17]
    lens = [pool[int(i)] for i in torch.randint(0, len(pool), (64,), generator=g)]
    lens[:4] = [0, 1, 64, 300]
    Hk, Hv, d = 2, 4, 128
    cu, x, h0, (q, k, v, a, b) = _packed(lens, Hk, Hv, d, torch.bfloat16, 95)
    o, ht = G.gdn_chunk_fwd_varlen(q, k, v, a, b, x["A_log"], x["dt_bias"], h0, cu,
                                   out_f32=True)
    assert G.gdn_status() == 0
    for i in range(len(lens)):
        s0, s1 = cu[i], cu[i + 1]
        sl = lambda t: t[s0:s1][None]
        o1, h1 = G.gdn_chunk_fwd(sl(q), sl(k), sl(v), sl(a), sl(b), x["A_log"], x["dt_bias"],
                                 h0[i:i + 1], out_f32=True)
        assert torch.equal(o[s0:s1], o1[0]) and torch.equal(ht[i], h1[0]), i
        if i < 6:
            ro, rht = O.gdn_fwd(cpu(sl(q)), cpu(sl(k)), cpu(sl(v)), cpu(sl(a)), cpu(sl(b)),
                                cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(h0[i:i + 1]))
            if s1 > s0:
                assert rel_err(o[s0:s1], ro[0]) <= TOL[torch.bfloat16]
            assert rel_err(ht[i], rht[0]) <= TOL[torch.bfloat16]


def test_varlen_more_sequences_than_one_launch_pair_takes():
    """With Hv = 64 one launch pair takes 65535 // 64 = 1023 sequences: 1100 short
    sequences run as two groups, each sequence's result that of its own call."""
    lens = [1 + (i % 3) for i in range(1100)]
    Hk, Hv, d = 16, 64, 128
    cu, x, h0, (q, k, v, a, b) = _packed(lens, Hk, Hv, d, torch.bfloat16, 96)
    o, ht = G.gdn_chunk_fwd_varlen(q, k, v, a, b, x["A_log"], x["dt_bias"], h0, cu,
                                   out_f32=True)
    assert G.gdn_status() == 0
    for i in (0, 1, 2, 1021, 1022, 1023, 1024, 1099):
        s0, s1 = cu[i], cu[i + 1]
        sl = lambda t: t[s0:s1][None]
        o1, h1 = G.gdn_chunk_fwd(sl(q), sl(k), sl(v), sl(a), sl(b), x["A_log"], x["dt_bias"],
                                 h0[i:i + 1], out_f32=True)
        assert torch.equal(o[s0:s1], o1[0]) and torch.equal(ht[i], h1[0]), i
