import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


# Collection order: the parity and unit files first (in file-name order), then
# the files whose failure should not stop them under -x, and the no-allocation
# entry point's test last of all.
LATE_FILES = ("test_empty_batch_gpu.py", "test_group_sizes_gpu.py", "test_wait_selftest_gpu.py")
LAST_FILE = "test_zz_no_alloc.py"


def _rank(item):
    name = os.path.basename(str(item.fspath))
    if name == LAST_FILE:
        return 2
    return 1 if name in LATE_FILES else 0


def pytest_collection_modifyitems(session, config, items):
    order = {id(it): i for i, it in enumerate(items)}
    items.sort(key=lambda it: (_rank(it), order[id(it)]))


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running oracle comparisons")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library through its Python binding (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sink_aware_sliding_head_b200 import flint_attn
    return flint_attn
