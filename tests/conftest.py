import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def pages_figures():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "pages_figures.json")) as f:
        return json.load(f)


def pytest_sessionstart(session):
    # The CUDA library is built in-tree (nvcc is part of the image on every box); this
    # only compiles when a source is newer than libcoact.so or the library is missing.
    build_library()


def build_library() -> str:
    """Runs co_activation_b200/build.py by path (importing the package needs the library)."""
    import runpy
    mod = runpy.run_path(os.path.join(ROOT, "co_activation_b200", "build.py"))
    return mod["build"]()
