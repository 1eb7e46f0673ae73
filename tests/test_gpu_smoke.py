"""The build entry point's smoke check (one small decode step against the oracle) runs as a GPU test too."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__ as entry
    entry.smoke()
