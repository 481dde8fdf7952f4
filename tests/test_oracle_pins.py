"""The fp64 oracle against its pins (CPU only).  See tests/_pins.py for what each pin fixes."""
import pytest

from tests import _pins


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_worked_example_fixture_shape():
    l, l_h, l_b, mats = _pins.load_worked_example()
    assert (l, l_h, l_b) == (6, 4, 3)
    assert set(mats) == {"H0", "H1"}
    assert all(len(row) == l_b for m in mats.values() for row in m)


def test_oracle_rejects_bad_args(oracle_lib):
    import numpy as np
    q = np.ones((1, 4, 6))
    with pytest.raises(AssertionError):
        oracle_lib.gated_fir(q, q, q, np.ones((4, 3)), 4)  # D % d_g != 0 -> wrong h rows
