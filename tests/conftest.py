import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Order in which the GPU test files run (a run that stops at the first failure
# has then covered the most basic parity first): the W4A4 path, its small-M
# kernels, then the other formats and variants, the measurement and failure
# checks, the guard bands around every output, and last the no-allocation
# entry point.  Files not listed keep their place between the host tests.
_FILE_ORDER = [
    "test_gpu_parity.py", "test_gpu_small_m.py", "test_gpu_int8.py", "test_gpu_groups.py", "test_gpu_asym.py",
    "test_gpu_measure.py", "test_gpu_failure.py", "test_zzz_canary.py", "test_zz_no_alloc.py",
]


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    rank = {name: i for i, name in enumerate(_FILE_ORDER)}

    def key(item):
        name = os.path.basename(str(item.fspath))
        return rank.get(name, -1)  # host-only files first, in collection order

    items[:] = [it for _, _, it in sorted((key(it), i, it) for i, it in enumerate(items))]
