"""The smoke check of the build entry point runs on cuda:0 and passes."""
import pytest

import __graft_entry__

pytestmark = pytest.mark.gpu


def test_smoke_entry_point(capsys):
    __graft_entry__.smoke()
    assert "smoke ok" in capsys.readouterr().out
