"""The bounded device waits of the tensor-core chunk kernels, made to expire on
purpose through the library's test hook (gdn_test_set_wait_fault): one hand-off
is withheld, so nothing is left in flight, and every wait polls a small number of
times.  The kernel must return (no hang, no CUDA error), gdn_check_status must
report GDN_ERR_TIMEOUT, and the next ordinary call on the same context must be
green.  No GPU fault is involved: the waits end by their own limit."""
import pytest
import torch

from gdn_synth import gdn2_inputs, gdn_inputs
from oracle import oracle as O
from tests.parity import cpu, rel_err

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"
TIMEOUT = -4


def _run_gdn(x):
    return G.gdn_chunk_fwd(x["q"], x["k"], x["v"], x["a"], x["b"], x["A_log"], x["dt_bias"],
                           x["h0"], out_f32=True)


@pytest.mark.parametrize("site", [1, 2], ids=["scan_state_handoff", "prep_tile_loads"])
def test_expired_wait_reports_timeout_and_context_stays_usable(site):
    x = gdn_inputs(2, 200, 2, 4, 128, torch.bfloat16, seed=71, device=DEV)
    try:
        G.gdn_test_set_wait_fault(site, 1 << 10)
        _run_gdn(x)  # the launch itself succeeds
        torch.cuda.synchronize()  # the kernels returned: no hang, no CUDA error
        assert G.gdn_status() == TIMEOUT
    finally:
        G.gdn_test_set_wait_fault(0, 0)
    assert G.gdn_status() == 0  # read-and-clear left a clean word
    o, ht = _run_gdn(x)
    assert G.gdn_status() == 0
    ro, rht = O.gdn_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b"]),
                        cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2


def test_expired_wait_in_the_shared_scan_of_gated_deltanet_2():
    """The Gated DeltaNet-2 path runs the same state scan: the same fault there."""
    x = gdn2_inputs(1, 150, 2, 128, torch.bfloat16, seed=72, device=DEV)
    args = (x["q"], x["k"], x["v"], x["a"], x["b_logit"], x["w_logit"], x["A_log"],
            x["dt_bias"], x["h0"])
    try:
        G.gdn_test_set_wait_fault(1, 1 << 10)
        G.gdn2_chunk_fwd(*args, out_f32=True)
        torch.cuda.synchronize()
        assert G.gdn_status() == TIMEOUT
    finally:
        G.gdn_test_set_wait_fault(0, 0)
    o, ht = G.gdn2_chunk_fwd(*args, out_f32=True)
    assert G.gdn_status() == 0
    ro, rht = O.gdn2_fwd(cpu(x["q"]), cpu(x["k"]), cpu(x["v"]), cpu(x["a"]), cpu(x["b_logit"]),
                         cpu(x["w_logit"]), cpu(x["A_log"]), cpu(x["dt_bias"]), cpu(x["h0"]))
    assert rel_err(o, ro) <= 2e-2 and rel_err(ht, rht) <= 2e-2


def test_unknown_fault_site_is_refused():
    with pytest.raises(G.GDNError):
        G.gdn_test_set_wait_fault(7, 0)
