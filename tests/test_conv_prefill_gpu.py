"""GPU parity of gdn_conv_prefill, the prefill-side causal depthwise conv1d
(kernel 4) + SiLU over the mixed [q | k | v] stream ("从 Full Attention 到 Gated
DeltaNet" section 10; "gated-deltanet-qwen3.5" section 因果卷积), called through
the C ABI and compared with the fp64 oracle on the same seeded inputs
(max|err|/RMS per tensor: 1e-4 for float32, 2e-2 for bf16; the conv window is a
byte copy and is compared bit for bit)."""
import numpy as np
import pytest
import torch

from gdn_synth import WORKLOADS, conv_prefill_inputs, gdn_inputs, workload_inputs
from oracle import oracle as O
from tests.parity import cpu, rel_err, rounding_ratio

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _split(y, Hk, Hv, d):
    B, T, _ = y.shape
    QK = Hk * d
    return (y[:, :, :QK].reshape(B, T, Hk, d), y[:, :, QK:2 * QK].reshape(B, T, Hk, d),
            y[:, :, 2 * QK:].reshape(B, T, Hv, d))


def _oracle(x, use_state):
    B, _, Cc = x["x"].shape
    cs = (cpu(x["conv_state"]).double().numpy().copy() if use_state else np.zeros((B, Cc, 3)))
    y = O.conv_prefill(cpu(x["x"]), cpu(x["conv_w"]), cs)
    return y, cs


@pytest.mark.parametrize("use_state", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [1, 2, 3, 17, 37, 100])
def test_conv_prefill_small(T, d, dtype, use_state):
    """Ragged token counts around the 16-token tile and the 3-token window."""
    B, Hk, Hv = 2, 2, 4
    x = conv_prefill_inputs(B, T, Hk, Hv, d, dtype, seed=40 + T, device=DEV)
    cs = x["conv_state"].clone() if use_state else None
    q, k, v = G.gdn_conv_prefill(x["x"], x["conv_w"], cs, Hk=Hk, Hv=Hv, dk=d, dv=d)
    y, r_cs = _oracle(x, use_state)
    rq, rk, rv = _split(y, Hk, Hv, d)
    if dtype == torch.bfloat16:  # one bf16 rounding of the exact conv + SiLU
        assert rounding_ratio(q, rq) <= 1 and rounding_ratio(k, rk) <= 1
        assert rounding_ratio(v, rv) <= 1
    else:
        assert rel_err(q, rq) <= 1e-4 and rel_err(k, rk) <= 1e-4 and rel_err(v, rv) <= 1e-4
    if use_state:
        np.testing.assert_array_equal(cpu(cs).double().numpy(), r_cs)


def test_conv_prefill_streams_bit_exact():
    """Two calls with the window carried in place give, bit for bit, one call over
    both (each output sees the same four inputs in the same float32 arithmetic)."""
    B, T1, T2, Hk, Hv, d = 2, 21, 40, 2, 4, 128
    x = conv_prefill_inputs(B, T1 + T2, Hk, Hv, d, torch.bfloat16, seed=47, device=DEV)
    cs1 = x["conv_state"].clone()
    q1, k1, v1 = G.gdn_conv_prefill(x["x"], x["conv_w"], cs1, Hk=Hk, Hv=Hv, dk=d, dv=d)
    cs2 = x["conv_state"].clone()
    qa, ka, va = G.gdn_conv_prefill(x["x"][:, :T1].contiguous(), x["conv_w"], cs2, Hk=Hk, Hv=Hv,
                                    dk=d, dv=d)
    qb, kb, vb = G.gdn_conv_prefill(x["x"][:, T1:].contiguous(), x["conv_w"], cs2, Hk=Hk, Hv=Hv,
                                    dk=d, dv=d)
    torch.testing.assert_close(torch.cat([qa, qb], 1), q1, rtol=0, atol=0)
    torch.testing.assert_close(torch.cat([ka, kb], 1), k1, rtol=0, atol=0)
    torch.testing.assert_close(torch.cat([va, vb], 1), v1, rtol=0, atol=0)
    torch.testing.assert_close(cs2, cs1, rtol=0, atol=0)


def test_conv_prefill_feeds_the_chunk_path():
    """conv prefill, then gdn_chunk_fwd (L2 norm in its prologue) on the tensor-core
    path, against the oracle's conv followed by the oracle's recurrence.  q, k and v
    cross the boundary between the two calls stored in the input dtype (bf16), so
    the oracle's conv outputs are rounded to bf16 at that same point."""
    B, T, Hk, Hv, d = 1, 100, 2, 4, 128
    x = conv_prefill_inputs(B, T, Hk, Hv, d, torch.bfloat16, seed=48, device=DEV)
    gates = gdn_inputs(B, T, Hk, Hv, d, torch.bfloat16, seed=49, device=DEV)
    cs = x["conv_state"].clone()
    q, k, v = G.gdn_conv_prefill(x["x"], x["conv_w"], cs, Hk=Hk, Hv=Hv, dk=d, dv=d)
    o, ht = G.gdn_chunk_fwd(q, k, v, gates["a"], gates["b"], gates["A_log"], gates["dt_bias"],
                            gates["h0"], out_f32=True)
    y, _ = _oracle(x, True)
    y = torch.from_numpy(y).bfloat16().double().numpy()
    rq, rk, rv = _split(y, Hk, Hv, d)
    ro, rht = O.gdn_fwd(rq, rk, rv, cpu(gates["a"]), cpu(gates["b"]), cpu(gates["A_log"]),
                        cpu(gates["dt_bias"]), cpu(gates["h0"]))
    assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2


def test_conv_prefill_full_size_sampled_tokens():
    """The mixed stream of the prefill_8k layer (B=1, T=8192, 16 key and 64 value
    heads, d=128, bf16): all channels of sampled tokens (the window's edge, tile
    edges, the last token) against the oracle's conv step from the window before
    each, and the final window bit for bit."""
    w = WORKLOADS["conv_prefill_8k"]
    x = workload_inputs(w, DEV)
    cs = x["conv_state"].clone()
    q, k, v = G.gdn_conv_prefill(x["x"], x["conv_w"], cs, Hk=w.Hk, Hv=w.Hv, dk=w.d, dv=w.d)
    torch.cuda.synchronize()
    xb = cpu(x["x"])[0]                               # [T, Cc] bf16
    cs0 = cpu(x["conv_state"])[0].double().numpy()    # [Cc, 3], index 2 newest

    def row(r):  # input r as float64; r < 0 reads the window before token 0
        return xb[r].double().numpy() if r >= 0 else cs0[:, r + 3]

    wcv = cpu(x["conv_w"])
    rng = np.random.default_rng(7)
    ts = sorted(set([0, 1, 2, 3, 15, 16, 17, w.T - 17, w.T - 16, w.T - 1] +
                    [int(t) for t in rng.integers(0, w.T, 40)]))
    QK = w.Hk * w.d
    qc, kc, vc = cpu(q)[0], cpu(k)[0], cpu(v)[0]
    got, ref = [], []
    for t in ts:
        win = np.ascontiguousarray(np.stack([row(t - 3), row(t - 2), row(t - 1)], 1)[None])
        xt = row(t).astype(np.float32)[None]
        ref.append(O.conv_step(xt, wcv, win)[0])
        got.append(torch.cat([qc[t].reshape(-1), kc[t].reshape(-1), vc[t].reshape(-1)]))
    got, ref = torch.stack(got), np.stack(ref)
    assert rounding_ratio(got, ref) <= 1
    assert rounding_ratio(got[:, :QK], ref[:, :QK]) <= 1
    last = np.stack([row(w.T - 3), row(w.T - 2), row(w.T - 1)], 1)
    np.testing.assert_array_equal(cpu(cs)[0].double().numpy(), last)
