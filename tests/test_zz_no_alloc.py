"""gdn_chunk_fwd_noalloc (GPU): the chunk forward with the library's fixed
64 MiB device scratch instead of a caller workspace.  It must give the same
bits as gdn_chunk_fwd with a workspace, match the oracle, allocate no device
memory, run workspace-free shapes unchanged and refuse sizes above its capacity
without launching anything."""
import pytest
import torch

from gdn_synth import gdn_inputs
from oracle import oracle as O
from tests.parity import TOL, cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

CAPACITY = 64 << 20


def _args(x):
    return (x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"], x["h0"])


def test_noalloc_same_bits_as_workspace_path_and_oracle():
    shape = (2, 300, 2, 4, 128)
    need = G.gdn_chunk_workspace_bytes(*shape, 128, torch.bfloat16)
    assert 0 < need <= CAPACITY
    x = gdn_inputs(*shape, torch.bfloat16, seed=31, device="cuda")
    o_ref, ht_ref = G.gdn_chunk_fwd(*_args(x))
    o = torch.empty_like(o_ref)
    ht = torch.empty_like(ht_ref)
    G.gdn_chunk_fwd_noalloc(*_args(x), o=o, ht=ht)  # first use reserves the static array
    torch.cuda.synchronize()
    n_alloc = torch.cuda.memory_stats()["allocation.all.allocated"]
    used = torch.cuda.memory_allocated()
    G.gdn_chunk_fwd_noalloc(*_args(x), o=o, ht=ht)
    torch.cuda.synchronize()
    assert torch.cuda.memory_stats()["allocation.all.allocated"] == n_alloc
    assert torch.cuda.memory_allocated() == used
    assert torch.equal(o, o_ref) and torch.equal(ht, ht_ref)
    # parity on the float32 output of the same path (the bar of the test suite)
    o32, ht32 = G.gdn_chunk_fwd_noalloc(*_args(x), out_f32=True)
    assert torch.equal(ht32, ht)
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    assert rel_err(o32, ro) <= TOL[torch.bfloat16] and rel_err(ht, rht) <= TOL[torch.bfloat16]
    assert torch.equal(o32.to(torch.bfloat16), o)


def test_noalloc_workspace_free_shapes_run_unchanged():
    x = gdn_inputs(1, 100, 1, 2, 128, torch.float32, seed=32, device="cuda")
    o, ht = G.gdn_chunk_fwd_noalloc(*_args(x))
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    assert rel_err(o, ro) <= 1e-4 and rel_err(ht, rht) <= 1e-4


def test_noalloc_refuses_sizes_above_capacity():
    shape = (1, 8192, 4, 16, 128)
    assert G.gdn_chunk_workspace_bytes(*shape, 128, torch.bfloat16) > CAPACITY
    x = gdn_inputs(*shape, torch.bfloat16, seed=33, device="cuda")
    o = torch.full((1, 8192, 16, 128), 7.0, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(G.GDNError) as e:
        G.gdn_chunk_fwd_noalloc(*_args(x), o=o)
    assert e.value.status == -5
    torch.cuda.synchronize()
    assert bool((o == 7.0).all())  # nothing was launched
