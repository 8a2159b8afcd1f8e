import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _library_is_stale() -> bool:
    pkg = os.path.join(ROOT, "hierarchical_sparse_attention_zha_b200")
    lib = os.path.join(pkg, "libzha.so")
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    srcs = [os.path.join(pkg, "csrc", f) for f in os.listdir(os.path.join(pkg, "csrc"))]
    srcs.append(os.path.join(ROOT, "include", "zha.h"))
    return any(os.path.getmtime(s) > t for s in srcs)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")
    if _library_is_stale():
        from hierarchical_sparse_attention_zha_b200 import build
        build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
