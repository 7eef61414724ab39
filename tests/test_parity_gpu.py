"""GPU parity: every entry point of libgdn.so, called through the C ABI, against
the fp64 oracle on the same seeded inputs (max|err|/RMS per tensor, raw: 1e-4 for
float32 inputs, 2e-2 for bf16 inputs).  For bf16 inputs the bar is applied to the
float32 output of the computation (GDN_OUT_F32), and the bf16 output of the same
call is checked bit for bit to be its round-to-nearest (see tests/parity.py)."""

import numpy as np
import pytest
import torch

from gdn_synth import WORKLOADS, decode_inputs, gdn2_inputs, gdn_inputs, workload_inputs
from oracle import oracle as O
from tests.parity import TOL, assert_bf16_store, cpu, rel_err, rounding_ratio

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _oracle_gdn(x, heads=None, **kw):
    return O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                     cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]), heads=heads, **kw)


def _gpu_gdn(x, **kw):
    """The chunk forward with float32 outputs unless out_f32=False is asked for."""
    kw.setdefault("out_f32", True)
    return G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                           x["h0"], **kw)


# ------------------------------------------------------------------ gate prep
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_gate_prep(dtype, d):
    x = gdn_inputs(2, 37, 2, 6, d, dtype, seed=11, device=DEV)
    qh, kh, g, beta = G.gdn_gate_prep(x["q"], x["k"], x["a"], x["b"], x["A_log"], x["dt_bias"])
    rq, rk, rg, rb = O.gate_prep(cpu(x["q"]), cpu(x["k"]), cpu(x["a"]), cpu(x["b"]),
                                 cpu(x["A_log"]), cpu(x["dt_bias"]))
    if dtype == torch.bfloat16:  # one final bf16 rounding of the normalised rows
        assert rounding_ratio(qh, rq) <= 1 and rounding_ratio(kh, rk) <= 1
    else:
        assert rel_err(qh, rq) <= 1e-4 and rel_err(kh, rk) <= 1e-4
    assert rel_err(g, rg) <= 1e-5 and rel_err(beta, rb) <= 1e-5


def test_gate_prep_in_place():
    x = gdn_inputs(1, 16, 2, 4, 128, torch.bfloat16, seed=12, device=DEV)
    rq, rk, _, _ = O.gate_prep(cpu(x["q"]), cpu(x["k"]), cpu(x["a"]), cpu(x["b"]),
                               cpu(x["A_log"]), cpu(x["dt_bias"]))
    q, k = x["q"].clone(), x["k"].clone()
    G.gdn_gate_prep(q, k, x["a"], x["b"], x["A_log"], x["dt_bias"], q_out=q, k_out=k)
    assert rounding_ratio(q, rq) <= 1 and rounding_ratio(k, rk) <= 1


# ------------------------------------------------------------ chunk prefill
def test_chunk_tiny_fp32_workload():
    """B=1, T=256, H=2, d=64, float32, zero initial state: bar 1e-4."""
    w = WORKLOADS["tiny_fp32"]
    x = workload_inputs(w, DEV)
    o, ht = _gpu_gdn(x)
    ro, rht = _oracle_gdn(x)
    assert rel_err(o, ro) <= 1e-4
    assert rel_err(ht, rht) <= 1e-4


SHAPES = [  # B, T, Hk, Hv, d
    (1, 1, 1, 1, 128), (1, 63, 1, 2, 128), (2, 64, 2, 2, 64), (1, 65, 2, 4, 128),
    (2, 100, 1, 4, 64), (1, 200, 2, 8, 128), (1, 384, 16, 64, 128), (3, 130, 2, 4, 128),
    (2, 1000, 2, 2, 128),
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_chunk_shapes(shape, dtype):
    B, T, Hk, Hv, d = shape
    x = gdn_inputs(B, T, Hk, Hv, d, dtype, seed=100 + T, device=DEV)
    o, ht = _gpu_gdn(x)
    assert o.dtype == torch.float32
    ro, rht = _oracle_gdn(x)
    assert rel_err(o, ro) <= TOL[dtype], rel_err(o, ro)
    assert rel_err(ht, rht) <= TOL[dtype], rel_err(ht, rht)
    if dtype == torch.bfloat16:
        o16, ht16 = _gpu_gdn(x, out_f32=False)
        assert o16.dtype == torch.bfloat16
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)  # the state does not depend on the output type


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_chunk_zero_initial_state_and_in_place_state(dtype):
    x = gdn_inputs(1, 130, 2, 4, 128, dtype, seed=5, device=DEV)
    x0 = dict(x, h0=None)
    o, ht = _gpu_gdn(x0)
    ro, rht = _oracle_gdn(x0)
    assert rel_err(o, ro) <= TOL[dtype] and rel_err(ht, rht) <= TOL[dtype]
    # ht aliasing h0: the state is updated in place
    h = x["h0"].clone()
    o2, ht2 = G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"],
                              x["dt_bias"], h, ht=h, out_f32=True)
    ro2, rht2 = _oracle_gdn(x)
    assert ht2.data_ptr() == h.data_ptr()
    assert rel_err(o2, ro2) <= TOL[dtype] and rel_err(h, rht2) <= TOL[dtype]


def test_chunk_workspace_reuse_and_size_check():
    """The workspace carries nothing from call to call: one NaN-filled buffer
    serves two different problems; a workspace one chunk-row short is refused."""
    shape = (2, 190, 2, 4, 128)
    need = G.gdn_chunk_workspace_bytes(*shape, 128, torch.bfloat16)
    assert need > 0
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)  # bf16 0xFFFF = NaN
    for seed in (21, 22):
        x = gdn_inputs(*shape, torch.bfloat16, seed=seed, device=DEV)
        o, ht = _gpu_gdn(x, workspace=ws)
        ro, rht = _oracle_gdn(x)
        assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2
    with pytest.raises(G.GDNError):
        _gpu_gdn(x, workspace=ws[: need - 16])


def test_chunk_empty_sequence_copies_state():
    x = gdn_inputs(2, 0, 2, 4, 128, torch.bfloat16, seed=6, device=DEV)
    o, ht = _gpu_gdn(x)
    assert o.shape == (2, 0, 4, 128)
    torch.testing.assert_close(ht, x["h0"], rtol=0, atol=0)
    o, ht = _gpu_gdn(dict(x, h0=None))
    assert torch.count_nonzero(ht).item() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_chunk_precomputed_gates_and_no_norm(dtype):
    """GDN_GATES_PRECOMPUTED with the oracle's own g, beta; and GDN_QK_L2NORM off
    with unit-norm q, k supplied by the caller."""
    x = gdn_inputs(1, 150, 2, 4, 128, dtype, seed=8, device=DEV)
    q = torch.nn.functional.normalize(x["q"].float(), dim=-1).to(dtype)
    k = torch.nn.functional.normalize(x["k"].float(), dim=-1).to(dtype)
    _, _, g, beta = O.gate_prep(cpu(x["q"]), cpu(x["k"]), cpu(x["a"]), cpu(x["b"]),
                                cpu(x["A_log"]), cpu(x["dt_bias"]))
    g32 = torch.from_numpy(g).float().to(DEV)
    b32 = torch.from_numpy(beta).float().to(DEV)
    scale = 128 ** -0.5
    o, ht = G.gdn_chunk_fwd(q, k, x["v"], g32, b32, None, None, x["h0"], l2norm=False,
                            gates_precomputed=True, scale=scale, out_f32=True)
    ro, rht = O.gdn_fwd(cpu(q), cpu(k), cpu(x["v"]), cpu(g32), cpu(b32), h0=cpu(x["h0"]),
                        scale=scale, l2norm=False, gates_given=True)
    assert rel_err(o, ro) <= TOL[dtype] and rel_err(ht, rht) <= TOL[dtype]


def test_chunk_streaming_split():
    """Two calls with the state carried equal the oracle's single pass."""
    x = gdn_inputs(1, 300, 2, 4, 128, torch.bfloat16, seed=9, device=DEV)
    p1 = {n: (t[:, :130] if n in ("q", "k", "v", "a", "b") else t) for n, t in x.items()}
    p2 = {n: (t[:, 130:].contiguous() if n in ("q", "k", "v", "a", "b") else t)
          for n, t in x.items()}
    o1, h1 = _gpu_gdn({**p1, **{n: p1[n].contiguous() for n in ("q", "k", "v", "a", "b")}})
    o2, h2 = _gpu_gdn(dict(p2, h0=h1))
    ro, rht = _oracle_gdn(x)
    assert rel_err(torch.cat([o1, o2], 1), ro) <= 2e-2
    assert rel_err(h2, rht) <= 2e-2


def _sampled_heads(B, Hv, n, seed):
    rng = np.random.default_rng(seed)
    return sorted(rng.choice(B * Hv, size=n, replace=False).tolist())


@pytest.mark.parametrize("name,n_heads", [("prefill_8k", 6), ("prefill_b8_16k", 2),
                                          ("prefill_128k", 2)])
def test_chunk_full_size_sampled_heads(name, n_heads):
    """Full-size workloads in the benchmark's launch configuration (bf16 output); the
    same call with float32 output carries the parity bar, the bf16 output is its
    rounding bit for bit; the oracle recomputes a sample of (batch, value head)
    scans end to end."""
    w = WORKLOADS[name]
    x = workload_inputs(w, DEV)
    o16, ht16 = _gpu_gdn(x, out_f32=False)
    o, ht = _gpu_gdn(x)
    assert torch.equal(ht16, ht)
    heads = _sampled_heads(w.B, w.Hv, n_heads, seed=w.seed)
    G_ = w.Hv // w.Hk
    errs = []
    for bh in heads:
        b, hv = divmod(bh, w.Hv)
        hk = hv // G_
        assert_bf16_store(o16[b, :, hv], o[b, :, hv])
        sub = {"q": x["q"][b:b + 1, :, hk:hk + 1], "k": x["k"][b:b + 1, :, hk:hk + 1],
               "v": x["v"][b:b + 1, :, hv:hv + 1], "a": x["a"][b:b + 1, :, hv:hv + 1],
               "b": x["b"][b:b + 1, :, hv:hv + 1], "A_log": x["A_log"][hv:hv + 1],
               "dt_bias": x["dt_bias"][hv:hv + 1], "h0": x["h0"][b:b + 1, hv:hv + 1]}
        ro, rht = _oracle_gdn(sub)
        errs.append((rel_err(o[b, :, hv], ro[0, :, 0]), rel_err(ht[b, hv], rht[0, 0])))
    assert max(max(e) for e in errs) <= 2e-2, errs
    assert torch.isfinite(o16.float()).all() and torch.isfinite(ht).all()


# ------------------------------------------------------------------ decode
def _decode_run(N, steps, Hk, Hv, d, dtype, seed, use_conv=True, seqs=None):
    """`steps` decode steps with float32 outputs (parity against the oracle) and, for
    bf16 inputs, the same steps on a copy of the states with bf16 outputs, which must
    be the round-to-nearest of the float32 ones, with identical states."""
    x = decode_inputs(N, steps, Hk, Hv, d, dtype, seed, device=DEV)
    conv_state = x["conv_state"].clone()
    state = x["state"].clone()
    twin = dtype == torch.bfloat16
    cs16, st16 = conv_state.clone(), state.clone()
    sel = list(range(N)) if seqs is None else seqs
    r_cs = cpu(x["conv_state"])[sel].double().numpy().copy()
    r_S = cpu(x["state"])[sel].double().numpy().copy()
    errs_o = []
    for t in range(steps):
        cw = x["conv_w"] if use_conv else None
        o = G.gdn_recurrent_step(x["x"][t], cw, conv_state, x["a"][t], x["b"][t], x["A_log"],
                                 x["dt_bias"], state, Hk=Hk, Hv=Hv, dk=d, dv=d, out_f32=True)
        if twin:
            o16 = G.gdn_recurrent_step(x["x"][t], cw, cs16, x["a"][t], x["b"][t], x["A_log"],
                                       x["dt_bias"], st16, Hk=Hk, Hv=Hv, dk=d, dv=d)
            assert_bf16_store(o16, o)
        ro = O.decode_step(cpu(x["x"][t]), cpu(x["conv_w"]) if use_conv else None,
                           cpu(x["a"][t]), cpu(x["b"][t]), cpu(x["A_log"]), cpu(x["dt_bias"]),
                           r_cs, r_S, Hk=Hk, Hv=Hv, dk=d, dv=d, seqs=seqs)
        errs_o.append(rel_err(o[sel], ro))
    if twin:
        assert torch.equal(st16, state) and torch.equal(cs16, conv_state)
    return x, conv_state, state, r_cs, r_S, errs_o


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small(dtype, d):
    x, cs, S, r_cs, r_S, errs = _decode_run(3, 5, 2, 4, d, dtype, seed=21)
    assert max(errs) <= TOL[dtype], errs
    assert rel_err(S, r_S) <= TOL[dtype]
    # the conv window is a byte copy: bit-exact
    np.testing.assert_array_equal(cpu(cs).double().numpy(), r_cs)


def test_decode_without_conv():
    x, cs, S, r_cs, r_S, errs = _decode_run(2, 3, 2, 4, 128, torch.bfloat16, seed=22,
                                            use_conv=False)
    assert max(errs) <= 2e-2
    assert rel_err(S, r_S) <= 2e-2
    torch.testing.assert_close(cs, x["conv_state"], rtol=0, atol=0)  # untouched


def test_decode_full_size_sampled_sequences():
    """256 sequences x 64 steps, Qwen3.5 head layout; oracle on 3 sequences."""
    w = WORKLOADS["decode_256"]
    seqs = [0, 97, 255]
    x, cs, S, r_cs, r_S, errs = _decode_run(w.B, w.steps, w.Hk, w.Hv, w.d, w.dtype, w.seed,
                                            seqs=seqs)
    assert max(errs) <= 2e-2, max(errs)
    assert rel_err(S[seqs], r_S) <= 2e-2
    np.testing.assert_array_equal(cpu(cs)[seqs].double().numpy(), r_cs)


# ------------------------------------------------------------------ GDN-2
def _oracle_gdn2(x, heads=None):
    return O.gdn2_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b_logit"]),
                      cpu(x["w_logit"]), cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]),
                      heads=heads)


def _gpu_gdn2(x, **kw):
    """The Gated DeltaNet-2 forward with float32 outputs unless out_f32=False."""
    kw.setdefault("out_f32", True)
    return G.gdn2_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b_logit"], x["w_logit"],
                            x["A_log"], x["dt_bias"], x["h0"], **kw)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 1, 1, 128), (1, 63, 1, 128), (1, 70, 2, 128),
                                   (2, 129, 2, 64), (1, 256, 4, 128), (3, 200, 2, 128),
                                   (1, 1000, 1, 128)])
def test_gdn2_shapes(shape, dtype):
    B, T, H, d = shape
    x = gdn2_inputs(B, T, H, d, dtype, seed=300 + T, device=DEV)
    o, ht = _gpu_gdn2(x)
    ro, rht = _oracle_gdn2(x)
    assert rel_err(o, ro) <= TOL[dtype], rel_err(o, ro)
    assert rel_err(ht, rht) <= TOL[dtype], rel_err(ht, rht)
    if dtype == torch.bfloat16:
        o16, ht16 = _gpu_gdn2(x, out_f32=False)
        assert_bf16_store(o16, o)
        assert torch.equal(ht16, ht)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gdn2_zero_and_in_place_state(dtype):
    x = gdn2_inputs(1, 150, 2, 128, dtype, seed=41, device=DEV)
    x0 = dict(x, h0=None)
    o, ht = _gpu_gdn2(x0)
    ro, rht = _oracle_gdn2(x0)
    assert rel_err(o, ro) <= TOL[dtype] and rel_err(ht, rht) <= TOL[dtype]
    h = x["h0"].clone()
    o2, ht2 = _gpu_gdn2(dict(x, h0=h), ht=h)
    ro2, rht2 = _oracle_gdn2(x)
    assert ht2.data_ptr() == h.data_ptr()
    assert rel_err(o2, ro2) <= TOL[dtype] and rel_err(h, rht2) <= TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gdn2_precomputed_gates_and_no_norm(dtype):
    """GDN_GATES_PRECOMPUTED: a = per-channel log-decay, b / w = gate values (float32);
    GDN_QK_L2NORM off with unit-norm q, k from the caller."""
    x = gdn2_inputs(2, 140, 2, 128, dtype, seed=42, device=DEV)
    q = torch.nn.functional.normalize(x["q"].float(), dim=-1).to(dtype)
    k = torch.nn.functional.normalize(x["k"].float(), dim=-1).to(dtype)
    a = cpu(x["a"]).double()
    g = -torch.exp(cpu(x["A_log"]).double()) * torch.nn.functional.softplus(
        a + cpu(x["dt_bias"]).double())
    bg = torch.sigmoid(cpu(x["b_logit"]).double())
    wg = torch.sigmoid(cpu(x["w_logit"]).double())
    g32, b32, w32 = (t.float().to(DEV) for t in (g, bg, wg))
    scale = 128 ** -0.5
    o, ht = G.gdn2_chunk_fwd(q, k, x["v"], g32, b32, w32, None, None, x["h0"], scale=scale,
                             l2norm=False, gates_precomputed=True, out_f32=True)
    ro, rht = O.gdn2_fwd(cpu(q), cpu(k), cpu(x["v"]), cpu(g32), cpu(b32), cpu(w32),
                         h0=cpu(x["h0"]), scale=scale, l2norm=False, gates_given=True)
    assert rel_err(o, ro) <= TOL[dtype] and rel_err(ht, rht) <= TOL[dtype]


def test_gdn2_workspace_reuse_and_size_check():
    shape = (2, 190, 2, 128)
    need = G.gdn2_chunk_workspace_bytes(*shape, 128, torch.bfloat16)
    assert need > 0
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device=DEV)  # fp16 / f32 NaN patterns
    for seed in (43, 44):
        x = gdn2_inputs(*shape, torch.bfloat16, seed=seed, device=DEV)
        o, ht = _gpu_gdn2(x, workspace=ws)
        ro, rht = _oracle_gdn2(x)
        assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2
    with pytest.raises(G.GDNError):
        _gpu_gdn2(x, workspace=ws[: need - 16])


def test_gdn2_full_size_sampled_heads():
    w = WORKLOADS["gdn2_b4_4k"]
    x = workload_inputs(w, DEV)
    o16, ht16 = _gpu_gdn2(x, out_f32=False)  # the benchmark's launch configuration
    o, ht = _gpu_gdn2(x)
    assert torch.equal(ht16, ht)
    heads = _sampled_heads(w.B, w.Hv, 4, seed=w.seed)
    ro, rht = _oracle_gdn2(x, heads=heads)
    for i, bh in enumerate(heads):
        b, h = divmod(bh, w.Hv)
        assert_bf16_store(o16[b, :, h], o[b, :, h])
        assert rel_err(o[b, :, h], ro[i]) <= 2e-2
        assert rel_err(ht[b, h], rht[i]) <= 2e-2
