"""The smoke entry point (one small pass of every part of the hot path,
checked against the oracle) runs clean on the GPU."""

import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__
    __graft_entry__.smoke()
