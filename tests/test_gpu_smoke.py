"""The package's smoke entry point (one decode on cuda:0 checked against the
fp64 oracle) runs clean on the device."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__
    __graft_entry__.smoke()
