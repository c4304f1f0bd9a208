import os
import pathlib
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture
def repo_tmp(request):
    """A scratch directory inside the repository (under the git-ignored .pytest_cache)."""
    d = os.path.join(ROOT, ".pytest_cache", "scratch", request.node.name.replace("/", "_"))
    shutil.rmtree(d, ignore_errors=True)
    os.makedirs(d)
    return pathlib.Path(d)
