import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    """A fresh checkout has no libgdn.so yet: build it (the tests load it through the
    package, which refuses to import without it)."""
    lib = os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "libgdn.so")
    if os.path.exists(lib):
        return
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "gdn_b200_build", os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


# The parity tests of the newest entry points run after all the others, so that a
# run that stops at its first failure (-x) has already reported the rest.
_RUN_LAST = ("test_kda_gpu.py", "test_rmsnorm_gated_gpu.py", "test_varlen_gpu.py",
             "test_gated_norm_fused_gpu.py", "test_bwd_gpu.py")


def pytest_collection_modifyitems(session, config, items):
    def rank(it):
        name = os.path.basename(str(it.fspath))
        if name == "test_zz_no_alloc.py":  # the no-allocation entry point's test: always last
            return 2
        return 1 if name in _RUN_LAST else 0
    items.sort(key=rank)  # stable


try:
    import pytest
    import torch
    _CUDA = torch.cuda.is_available()
except Exception:  # noqa: BLE001
    _CUDA = False

if _CUDA:
    @pytest.fixture(autouse=True)
    def _device_status_clean(request):
        """Every GPU test starts and ends with a clean device status word: a set
        GDN_ERR_RANGE or GDN_ERR_TIMEOUT bit left by any call of the test (the word is
        sticky) fails the test that caused it.  Tests that provoke one on purpose
        read it themselves, which clears it."""
        if request.node.get_closest_marker("gpu") is None:
            yield
            return
        import gated_deltanet_sequence_gdn_b200 as G
        before = G.gdn_status()
        assert before == 0, f"device status {before} left by an earlier test"
        yield
        after = G.gdn_status()
        assert after == 0, f"device status {after} after the test (-4 timeout, -6 range)"


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")
