"""The CPU oracle against its pins (closed forms, invariants, library special
cases, finite differences). No GPU."""
import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_default_positions_restart_per_batch_row():
    m = oracle.positions(None, 3, 5)
    assert m.tolist() == [0, 1, 2, 3, 4] * 3
    ids = np.array([[4, 0, 1], [2, 2, 7]], dtype=np.int32)
    assert oracle.positions(ids, 2, 3).tolist() == [4, 0, 1, 2, 2, 7]


def test_inv_freq_entry_point(orc):
    assert orc.inv_freq(0, 64, 1e6) == 1.0
    assert abs(orc.inv_freq(32, 64, 1e6) - 1e-6) < 1e-21
