import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (runs the CUDA library)")
    config.addinivalue_line("markers", "slow: full-size parity cases")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library, loaded through its Python binding (fails loudly if absent)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import token_level_top_hs2_b200 as hs2
    hs2.load()
    return hs2
