import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_collection_modifyitems(config, items):
    # A run that selects GPU tests on a machine without a GPU should fail loudly, not skip:
    # the product has no CPU fallback. Nothing to do here; the gpu fixture checks it.
    pass


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    return torch.device("cuda:0")


@pytest.fixture(scope="session")
def sf(cuda):
    """The CUDA library through its Python binding (fails loudly if it is not built)."""
    from masked_optimizer_step_b200 import binding
    binding.load()
    return binding
