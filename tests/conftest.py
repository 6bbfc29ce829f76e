import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    # the C-ABI library is a build artefact: compile it (sm_100a, nvcc cross-compiles
    # without a GPU) when a checkout does not have it yet; an existing one is used as is
    from block_diffusion_lm_masked_b200 import build as B
    if not os.path.exists(B.LIB):
        B.build()
    # the C++ oracle likewise (test infrastructure; rebuilt when its source is newer)
    from oracle import build as OB
    OB.build()


def golden_path(name):
    return os.path.join(ROOT, "tests", "golden", name)
