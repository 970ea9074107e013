"""Shared pytest configuration: the ``gpu`` marker and the repository root on sys.path."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libtq.so")


def build_lib():
    """Compiles libtq.so in-tree if stale (loads the build script by path, so a stale
    library is never imported first), then returns the imported package."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_tq_build", os.path.join(ROOT, "embedding_vector_quantization_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import embedding_vector_quantization_b200 as tq
    return tq
