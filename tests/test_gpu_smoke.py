"""The entry point the round-end checks call: one small decode step per format family on
cuda:0 through the public API, checked against the fp64 oracle."""
import pytest


@pytest.mark.gpu
def test_smoke_entry_point():
    import __graft_entry__ as g
    g.smoke()
