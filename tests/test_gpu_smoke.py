"""The package entry point's smoke run (one small layer forward on cuda:0 against the oracle)."""
import pytest


@pytest.mark.gpu
def test_entry_point_smoke(capsys):
    import __graft_entry__ as entry
    entry.smoke()
    assert "smoke ok" in capsys.readouterr().out
