import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; parity tests through the C-ABI")
    config.addinivalue_line("markers", "slow: long-running CPU test")


# GPU modules in the order they were established: under -x, a failure in a newer module does not
# keep the older suites from running (and being reported).  Modules not listed (CPU tests) come
# first, in their own order.
# The no-alloc entry point's module comes last of all, so that a failure there cannot stop any other
# suite under -x.
_GPU_MODULE_ORDER = ("test_gpu_parity.py", "test_gpu_full_tensor.py", "test_gpu_decode.py",
                     "test_gpu_decode_tiles.py", "test_gpu_neighbors.py", "test_gpu_bwd.py", "test_gpu_bwd_tc.py",
                     "test_zz_no_alloc.py")


def pytest_collection_modifyitems(session, config, items):
    def rank(item):
        name = os.path.basename(str(item.fspath))
        return _GPU_MODULE_ORDER.index(name) if name in _GPU_MODULE_ORDER else -1
    items.sort(key=rank)  # stable: the order inside each module is unchanged
