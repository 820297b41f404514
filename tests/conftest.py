import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def bra_lib():
    """The built C-ABI library (compiled on demand from the in-tree sources)."""
    from vision_transformer_sparse_b200 import build as vbuild
    vbuild.build_library()
    from vision_transformer_sparse_b200 import bra
    return bra.lib()
