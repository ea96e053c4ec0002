import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def product():
    """The product package with its library built (fails loudly if the build fails)."""
    from block_sparse_attention_29_b200 import build as b
    b.build()
    import block_sparse_attention_29_b200 as sa
    sa._lib.lib()
    return sa


@pytest.fixture(scope="session")
def cuda(product):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA GPU required for tests marked gpu")
    torch.cuda.init()
    return torch.device("cuda:0")
