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
_RUN_LAST = ("test_kda_gpu.py", "test_rmsnorm_gated_gpu.py", "test_varlen_gpu.py")


def pytest_collection_modifyitems(session, config, items):
    items.sort(key=lambda it: os.path.basename(str(it.fspath)) in _RUN_LAST)  # stable


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")
