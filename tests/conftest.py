import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100) GPU and the built CUDA library")
    config.addinivalue_line(
        "markers", "slow: long CPU or GPU test (full-size workloads)")


@pytest.fixture(scope="session")
def lib():
    """The GPU library through its Python binding; skips cleanly when no GPU
    is present (the -m gpu run happens on a GPU machine)."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_13_b200 as g
    return g


def pytest_sessionstart(session):
    """With GPTQ_ORACLE_MUTANT set (only by test_oracle_mutants.py, in a
    child process), plant that mistake in the oracle before any test runs."""
    name = os.environ.get("GPTQ_ORACLE_MUTANT")
    if name:
        sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
        import oracle_mutants
        oracle_mutants.apply(name)
