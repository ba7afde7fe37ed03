import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")

# Build the two native libraries in-tree if they are missing or stale (nvcc and gcc
# cross-compile without a GPU).  The CUDA library is never replaced by a fallback: if it
# cannot be built, importing the binding fails.
from oracle.build import build_oracle  # noqa: E402
from qat_nvfp4_b200.build import build_library  # noqa: E402

build_oracle()
build_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_collection_modifyitems(config, items):
    # GPU tests are only meaningful with a device; on a CPU-only host they are skipped
    # when selected explicitly (the default CPU run deselects them with -m "not gpu").
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this host")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN
