import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    """A tree without the CUDA library (a fresh checkout) gets it built
    before collection: the test modules import the package, which needs it.
    The builder is loaded by its path, since importing the package itself
    needs the library."""
    if os.path.exists(os.path.join(ROOT, "quantized_expert_gemv_b200", "libfmoe.so")):
        return
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fmoe_library_build", os.path.join(ROOT, "quantized_expert_gemv_b200", "build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size oracle work)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
