"""The package's smoke check (one small GDP decode step, a varlen prefill and its
backward on cuda:0, each against the oracle) runs as part of the GPU suite."""
import os
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_smoke_entry_point():
    sys.path.insert(0, ROOT)
    import __graft_entry__
    __graft_entry__.smoke()
