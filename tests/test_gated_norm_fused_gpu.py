"""GPU parity of the gated RMSNorm fused into the output store of the chunk
forward (gdn_chunk_fwd_gated_norm) and of the decode step
(gdn_recurrent_step_gated_norm): o = core / sqrt(mean(core^2) + eps) * w * SiLU(z)
per (token, value head) ("gated-deltanet-qwen3.5", 输出门控与 RMSNorm), against the
oracle's gated RMSNorm applied to the oracle's recurrence, on the same seeded
inputs (max|err|/RMS raw on float32 outputs: 2e-2 for bf16 inputs, 1e-4 for
float32; bf16 outputs checked bit for bit to be the rounding of the float32 ones)."""
import numpy as np
import pytest
import torch

from gdn_synth import WORKLOADS, decode_inputs, gdn_inputs, workload_inputs
from oracle import oracle as O
from tests.parity import TOL, assert_bf16_store, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _gate(B, T, Hv, dv, dtype, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    z = torch.randn(B, T, Hv, dv, generator=g).to(dtype)
    w = 0.5 + torch.rand(dv, generator=g)
    return z.to(DEV), w.to(DEV)


def _chunk(x, z, w, eps, **kw):
    return G.gdn_chunk_fwd_gated_norm(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                      x["dt_bias"], x["h0"], z, w, eps=eps, **kw)


def _ref(x, z, w, eps, heads=None):
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]), heads=heads)
    return O.rmsnorm_gated(ro, cpu(z).double().numpy(), cpu(w).double().numpy(), eps=eps), rht


SHAPES = [(1, 1, 1, 1, 128), (1, 65, 1, 2, 128), (2, 130, 2, 4, 128), (1, 300, 2, 8, 128),
          (3, 100, 1, 1, 128), (2, 64, 2, 2, 64), (1, 130, 2, 4, 64)]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_chunk_gated_norm_matches_oracle(shape, dtype):
    B, T, Hk, Hv, d = shape
    x = gdn_inputs(B, T, Hk, Hv, d, dtype, seed=500 + T + d, device=DEV)
    z, w = _gate(B, T, Hv, d, dtype, seed=600 + T)
    eps = 1e-6
    o, ht = _chunk(x, z, w, eps, out_f32=True)
    ro, rht = _ref(x, z, w, eps)
    assert rel_err(o, ro) <= TOL[dtype], rel_err(o, ro)
    assert rel_err(ht, rht) <= TOL[dtype]
    if dtype == torch.bfloat16 and d == 128:  # fused: the bf16 store rounds the same rows
        o16, ht16 = _chunk(x, z, w, eps)
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)


def test_chunk_gated_norm_state_and_flags():
    """The state is that of gdn_chunk_fwd bit for bit; precomputed gates without the
    norm of q / k; a large eps and an all-zero gate row (output zero there)."""
    B, T, Hk, Hv, d = 1, 150, 2, 4, 128
    x = gdn_inputs(B, T, Hk, Hv, d, torch.bfloat16, seed=510, device=DEV)
    z, w = _gate(B, T, Hv, d, torch.bfloat16, seed=511)
    z[0, 7, 1] = 0.0
    o, ht = _chunk(x, z, w, 0.5, out_f32=True)
    _, ht_plain = G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                                  x["dt_bias"], x["h0"], out_f32=True)
    assert torch.equal(ht, ht_plain)
    ro, _ = _ref(x, z, w, 0.5)
    assert rel_err(o, ro) <= 2e-2
    assert bool((o[0, 7, 1] == 0).all())


def test_chunk_gated_norm_full_size_sampled_heads():
    """prefill_8k (B=1, T=8192, 16 key / 64 value heads, d=128, bf16) in the bench's
    launch configuration (bf16 output) and with float32 output; sampled heads."""
    w_ = WORKLOADS["prefill_8k"]
    x = workload_inputs(w_, DEV)
    z, w = _gate(w_.B, w_.T, w_.Hv, w_.d, w_.dtype, seed=512)
    o16, ht16 = _chunk(x, z, w, 1e-6)
    o, ht = _chunk(x, z, w, 1e-6, out_f32=True)
    assert torch.equal(ht16, ht)
    rng = np.random.default_rng(5)
    G_ = w_.Hv // w_.Hk
    for hv in sorted(rng.choice(w_.Hv, size=3, replace=False).tolist()):
        hk = hv // G_
        sub = {"q": x["q"][:, :, hk:hk + 1], "k": x["k"][:, :, hk:hk + 1],
               "v": x["v"][:, :, hv:hv + 1], "a": x["a"][:, :, hv:hv + 1],
               "b": x["b"][:, :, hv:hv + 1], "A_log": x["A_log"][hv:hv + 1],
               "dt_bias": x["dt_bias"][hv:hv + 1], "h0": x["h0"][:, hv:hv + 1]}
        ro, _ = _ref(sub, z[:, :, hv:hv + 1], w, 1e-6)
        assert rel_err(o[:, :, hv:hv + 1], ro) <= 2e-2
        assert_bf16_store(o16[:, :, hv], o[:, :, hv])


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_gated_norm_matches_oracle(dtype, d):
    N, steps, Hk, Hv = 3, 4, 2, 4
    x = decode_inputs(N, steps, Hk, Hv, d, dtype, seed=520 + d, device=DEV)
    g = torch.Generator().manual_seed(521)
    z = torch.randn(steps, N, Hv, d, generator=g).to(dtype).to(DEV)
    w = (0.5 + torch.rand(d, generator=g)).to(DEV)
    cs, S = x["conv_state"].clone(), x["state"].clone()
    cs16, S16 = cs.clone(), S.clone()
    r_cs = cpu(x["conv_state"]).double().numpy().copy()
    r_S = cpu(x["state"]).double().numpy().copy()
    for t in range(steps):
        o = G.gdn_recurrent_step_gated_norm(x["x"][t], x["conv_w"], cs, x["a"][t], x["b"][t],
                                            x["A_log"], x["dt_bias"], S, z[t], w, Hk=Hk, Hv=Hv,
                                            dk=d, dv=d, out_f32=True)
        ro = O.decode_step(cpu(x["x"][t]), cpu(x["conv_w"]), cpu(x["a"][t]), cpu(x["b"][t]),
                           cpu(x["A_log"]), cpu(x["dt_bias"]), r_cs, r_S, Hk=Hk, Hv=Hv, dk=d,
                           dv=d)
        ry = O.rmsnorm_gated(ro, cpu(z[t]).double().numpy(), cpu(w).double().numpy())
        assert rel_err(o, ry) <= TOL[dtype], (t, rel_err(o, ry))
        if dtype == torch.bfloat16:
            o16 = G.gdn_recurrent_step_gated_norm(x["x"][t], x["conv_w"], cs16, x["a"][t],
                                                  x["b"][t], x["A_log"], x["dt_bias"], S16,
                                                  z[t], w, Hk=Hk, Hv=Hv, dk=d, dv=d)
            assert_bf16_store(o16, o)
    assert rel_err(S, r_S) <= TOL[dtype]


def test_gated_norm_argument_checks():
    x = gdn_inputs(1, 64, 1, 2, 128, torch.bfloat16, seed=530, device=DEV)
    z, w = _gate(1, 64, 2, 128, torch.bfloat16, seed=531)
    with pytest.raises(G.GDNError) as e:
        _chunk(x, z, w, -1.0)
    assert e.value.status == -1
    with pytest.raises(G.GDNError) as e:  # eps above 1
        _chunk(x, z, w, 2.0)
    assert e.value.status == -1
