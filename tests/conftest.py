import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


@pytest.hookimpl(tryfirst=True)
def pytest_configure(config):
    # temporary paths of the tests stay inside the repository (a git-ignored folder)
    if config.option.basetemp is None:
        os.makedirs(os.path.join(ROOT, "_build"), exist_ok=True)
        config.option.basetemp = os.path.join(ROOT, "_build", "pytest")
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_sessionstart(session):
    """Build the CUDA library, the generator and the oracle if they are stale."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("_moe_cuda_build",
                                                  os.path.join(ROOT, "bit_dequant_expert_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=False)
