import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # The C-ABI library is a build artefact (not committed); build it in-tree
    # when it is missing or older than its sources.  nvcc cross-compiles for
    # sm_100a without a GPU.
    import importlib.util
    path = os.path.join(ROOT, "retrieval_sparse_attention_wave_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_wi_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
