import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running full-size case")
    # a fresh checkout has no library yet: build it in-tree (nvcc, sm_100a)
    lib = os.path.join(ROOT, "sparse_state_reuse_b200", "libditango.so")
    if not os.path.exists(lib):
        subprocess.run([sys.executable, os.path.join(ROOT, "sparse_state_reuse_b200", "build.py")],
                       check=True)


@pytest.fixture(scope="session")
def rng():
    import numpy as np
    return np.random.default_rng(1234)
