import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload (seconds to minutes)")


@pytest.fixture(scope="session")
def cuda_dev():
    """The CUDA device for GPU tests; skips when no GPU is visible, fails loudly when
    a GPU is present but the CUDA library was not built."""
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device visible")
    import nvfp4_w4a4_quantized_amax_b200 as nv  # raises if libnvfp4.so is missing

    nv.library()  # loads the shared library now
    return torch.device("cuda:0")
