import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


def pytest_sessionstart(session):
    """Build libtq4.so in-tree when it is missing or older than its sources
    (nvcc cross-compiles for sm_100a without a GPU)."""
    from compressed_paged_kv_tq4_b200 import build
    if build.needs_build():
        build.build()
