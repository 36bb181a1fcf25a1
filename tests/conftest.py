import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size shapes)")


def pytest_sessionstart(session):
    # libvc.so is built in-tree (nvcc cross-compiles without a GPU); a fresh checkout builds it
    # once here, so that the tests that load it find it.  The package itself still refuses to
    # import without it.
    if not os.path.exists(os.path.join(ROOT, "attention_frame_decode_b200", "libvc.so")):
        import importlib.util
        path = os.path.join(ROOT, "attention_frame_decode_b200", "build.py")
        spec = importlib.util.spec_from_file_location("vc_build", path)
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()


def gpu_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda():
    if not gpu_available():
        pytest.skip("no CUDA device")
    import torch
    return torch.device("cuda:0")
