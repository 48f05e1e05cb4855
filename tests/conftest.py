import ctypes
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# The oracle allocates many large temporaries.  glibc hands big blocks back to
# the kernel on free, so every new array page-faults afresh, which is slow on
# virtual machines.  Keep freed memory in the heap (test process only).
try:
    _libc = ctypes.CDLL("libc.so.6")
    _libc.mallopt(-3, 32 * 1024 * 1024)  # M_MMAP_THRESHOLD
    _libc.mallopt(-1, 2 ** 31 - 1)       # M_TRIM_THRESHOLD
except OSError:  # pragma: no cover - non-glibc hosts
    pass


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: oracle work of tens of seconds")


@pytest.fixture(scope="session")
def has_gpu():
    import torch
    return torch.cuda.is_available()
