"""GPU parity of gdn_rmsnorm_gated, the gated RMSNorm of the core output
("gated-deltanet-qwen3.5" section 输出门控与 RMSNorm: RMSNormGated(core_attn_out,
z)), called through the C ABI and compared with the fp64 oracle on the same
seeded inputs (max|err|/RMS: 1e-4 for float32, 2e-2 for bf16)."""
import pytest
import torch

from gdn_synth import WORKLOADS, rmsnorm_inputs, workload_inputs
from oracle import oracle as O
from tests.parity import cpu, rel_err, rounding_ratio

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_deltanet_sequence_gdn_b200 as G

DEV = "cuda"


def _check(y, ref, dtype):
    """float32: the raw 1e-4 bar; bf16 (the only output type): one final bf16
    rounding of the exact value per element (tests/parity.py)."""
    if dtype == torch.bfloat16:
        assert rounding_ratio(y, ref) <= 1, rounding_ratio(y, ref)
    else:
        assert rel_err(y, ref) <= 1e-4, rel_err(y, ref)


def _oracle(x, eps=1e-6):
    return O.rmsnorm_gated(cpu(x["o"]), cpu(x["z"]), cpu(x["weight"]), eps=eps)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 37, 3), (1, 100, 5)])
def test_rmsnorm_gated_small(shape, dv, dtype):
    """Row counts that are not a multiple of the 8 rows a CTA takes."""
    B, T, H = shape
    x = rmsnorm_inputs(B, T, H, dv, dtype, seed=60 + T, device=DEV)
    y = G.gdn_rmsnorm_gated(x["o"], x["z"], x["weight"])
    _check(y, _oracle(x), dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rmsnorm_gated_in_place_and_eps(dtype):
    """y written over o, a larger eps, and all-zero rows (output zero, no NaN)."""
    x = rmsnorm_inputs(2, 19, 4, 128, dtype, seed=67, device=DEV)
    x["o"][0, 3] = 0.0
    ref = _oracle(x, eps=0.25)
    o = x["o"].clone()
    G.gdn_rmsnorm_gated(o, x["z"], x["weight"], eps=0.25, y=o)
    _check(o, ref, dtype)
    assert bool((o[0, 3] == 0).all())


def test_rmsnorm_gated_full_size():
    """The core output of the prefill_8k layer: 8192 tokens x 64 value heads x 128."""
    w = WORKLOADS["rmsnorm_gated_8k"]
    x = workload_inputs(w, DEV)
    y = G.gdn_rmsnorm_gated(x["o"], x["z"], x["weight"])
    _check(y, _oracle(x), torch.bfloat16)
