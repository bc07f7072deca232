"""The package's smoke check (__graft_entry__.smoke) as a GPU test, so that a
change which breaks it shows up with the rest of the suite."""
import pytest

import __graft_entry__

pytestmark = pytest.mark.gpu


def test_smoke_passes():
    __graft_entry__.smoke()
