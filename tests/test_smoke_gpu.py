"""The round-trip check that `__graft_entry__.smoke()` runs on a fresh GPU
(every kernel family and the host-buffer entry point on small problems
against the oracle) must itself pass: run it as a test."""
import os
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_smoke_entry_point():
    import __graft_entry__

    __graft_entry__.smoke()
