"""Shared pytest setup: the ``gpu`` marker, the repository root on sys.path, and an in-tree build of
libtq.so when it is missing or older than its sources (nvcc cross-compiles without a GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built libtq")
    from kv_cache_vector_norm_b200 import _build
    if _build.needs_build():
        _build.build()
