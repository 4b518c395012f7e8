import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; run through the C-ABI library")
    config.addinivalue_line("markers", "slow: full-size workload parity on the GPU (minutes of oracle time)")


import pytest  # noqa: E402


@pytest.fixture
def force_kernel():
    """Setter for the bf16 forward kernel choice (fa_test_force_forward_kernel);
    the choice goes back to 'by problem size' when the test ends, pass or fail."""
    import tiled_exact_attention_fa_b200 as fa
    lib = fa.library()

    def set_kernel(which: int) -> None:
        assert lib.fa_test_force_forward_kernel(which) == fa.FA_OK

    yield set_kernel
    lib.fa_test_force_forward_kernel(0)
