"""The entry point's smoke run (one tiny CSA decode step on cuda:0 against the
float64 oracle) runs as a test too, so that a fault in it shows before the
entry point is called on its own."""
import pytest


@pytest.mark.gpu
def test_entry_point_smoke():
    import __graft_entry__
    __graft_entry__.smoke()
