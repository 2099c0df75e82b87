import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running GPU case at full workload size")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device; run it with -m gpu on a GPU host")
    return torch.device("cuda:0")


@pytest.fixture(autouse=True, scope="session")
def _attention_kernel_choice():
    """FP8PD_TEST_KERNEL=1|2 runs the whole suite with FP8PD_OPT_KERNEL set
    (1 = split kernel, 2 = tensor-memory kernel where it applies)."""
    k = os.environ.get("FP8PD_TEST_KERNEL")
    if k is not None:
        import fp8_paged_decode_split_b200 as F
        F.fp8pd_set_option(F.OPT_KERNEL, int(k))
    yield
