"""Shared pytest setup: the repo root and this folder are importable, and the
``gpu`` marker (tests that need a B200) is registered."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (an sm_100a B200)")
