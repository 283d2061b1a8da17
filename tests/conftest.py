import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def launch_overlap_mode():
    """ENTRO_TEST_OVERLAP=1 runs every GPU test with launch overlap on (the bench's mode)."""
    if os.environ.get("ENTRO_TEST_OVERLAP") != "1":
        yield
        return
    import huffman_decode_canonical_b200 as entro
    prev = entro.set_overlap(True)
    yield
    entro.set_overlap(prev)


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
