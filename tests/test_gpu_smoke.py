"""The package's smoke check (one small training step of both streams on cuda:0,
compared with the oracle) runs as part of the GPU suite, so that a change that
breaks it shows up in the same run as the parity tests."""
import pytest

pytestmark = pytest.mark.gpu


def test_smoke_entry_point():
    import __graft_entry__

    __graft_entry__.smoke()
