"""The entry point's smoke check (one decode-size layer against the oracle)
runs as a GPU test too, so that a change that breaks it shows up with the
rest of the suite."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__ as entry
    entry.smoke()
