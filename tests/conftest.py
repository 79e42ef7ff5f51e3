import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
# The mutation tests point this at a folder holding a deliberately broken copy
# of the oracle package, imported in place of the real one.
MUTANT = os.environ.get("MPZCH_ORACLE_PKG_PARENT")
if MUTANT:
    sys.path.insert(0, MUTANT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU check")
