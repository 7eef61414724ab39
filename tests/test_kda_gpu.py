"""GPU parity of gdn_kda_chunk_fwd: KDA, Gated DeltaNet-2 with one beta per
(token, head) for the erase and the write ("Gated DeltaNet-2", sections
标量绑定的数学表达 and 退化兼容性).  Compared with the oracle's literal KDA update
(the erase projection formed explicitly) on the same seeded inputs (max|err|/RMS,
raw: 1e-4 for float32 inputs, 2e-2 for bf16 inputs, on float32 outputs; the bf16
output is their rounding bit for bit), and bit for bit with gdn2_chunk_fwd on the
gates tiled by hand."""
import pytest
import torch

from gdn_synth import kda_inputs
from oracle import oracle as O
from tests.parity import TOL, assert_bf16_store, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _tiled(x, dk, dv):
    b = x["beta"][..., None].expand(*x["beta"].shape, dk).contiguous()
    w = x["beta"][..., None].expand(*x["beta"].shape, dv).contiguous()
    return b, w


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("B,T", [(1, 1), (2, 63), (1, 100)])
def test_kda_small(B, T, dtype, d):
    """The tensor-core path (bf16, d = 128) and the float32 path, ragged chunks."""
    x = kda_inputs(B, T, 2, d, dtype, seed=70 + T, device=DEV)
    o, ht = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                                x["dt_bias"], x["h0"], out_f32=True)
    if dtype == torch.bfloat16:
        o16, ht16 = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                                        x["dt_bias"], x["h0"])
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)
    ro, rht = O.kda_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["beta"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    assert rel_err(o, ro) <= TOL[dtype] and rel_err(ht, rht) <= TOL[dtype]


def test_kda_is_gdn2_on_tiled_gates_bit_for_bit():
    """The same kernels on the same gate values: logits in bf16, and precomputed
    float32 gates (log-decay and beta)."""
    B, T, H, d = 2, 130, 2, 128
    x = kda_inputs(B, T, H, d, torch.bfloat16, seed=77, device=DEV)
    b, w = _tiled(x, d, d)
    o1, h1 = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                                 x["dt_bias"], x["h0"])
    o2, h2 = G.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["a"], b, w, x["A_log"], x["dt_bias"],
                              x["h0"])
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    g = -torch.rand(B, T, H, d, device=DEV) * 0.5
    beta = torch.rand(B, T, H, device=DEV)
    xp = {"beta": beta}
    bp, wp = _tiled(xp, d, d)
    o3, h3 = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], g, beta, h0=x["h0"],
                                 gates_precomputed=True)
    o4, h4 = G.gdn2_chunk_fwd(x["q"], x["k"], x["v"], g, bp, wp, h0=x["h0"],
                              gates_precomputed=True)
    assert torch.equal(o3, o4) and torch.equal(h3, h4)


def test_kda_full_size_sampled_heads():
    """B=4, T=4096, 16 heads, d=128 (the Gated DeltaNet-2 bench shape); the oracle
    recomputes two (batch, head) pairs end to end on the tiled gates."""
    B, T, H, d = 4, 4096, 16, 128
    x = kda_inputs(B, T, H, d, torch.bfloat16, seed=1007, device=DEV)
    o16, ht16 = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                                    x["dt_bias"], x["h0"])
    o, ht = G.gdn_kda_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"],
                                x["dt_bias"], x["h0"], out_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(ht16, ht)
    b, w = _tiled(x, d, d)
    for bh in (0, 2 * H + 9):
        bi, h = divmod(bh, H)
        ro, rht = O.gdn2_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(b), cpu(w),
                             cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]), heads=[bh])
        assert_bf16_store(o16[bi, :, h], o[bi, :, h])
        assert rel_err(o[bi, :, h], ro[0]) <= 2e-2 and rel_err(ht[bi, h], rht[0]) <= 2e-2
