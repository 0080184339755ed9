import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the CUDA library")
    config.addinivalue_line("markers", "slow: large CPU oracle work")
    # Build the in-tree CUDA library (a no-op when it is current) and the C oracle
    # before collection imports them.
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_awq_b200_build", os.path.join(ROOT, "weight_only_quantization_awq_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    build_lib = mod.build
    import oracle
    build_lib()
    oracle.build()
