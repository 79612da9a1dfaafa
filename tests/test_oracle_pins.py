"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import oracle_pins as P


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_pool_rows_max_bound(orc):
    # T*k real rows + (tile-1) padding for each non-empty expert, rounded to the tile
    assert orc.pool_rows_max(8192, 8, 256, 128) == 65536 + 256 * 127
    assert orc.pool_rows_max(1, 1, 256, 128) == 128
    assert orc.pool_rows_max(0, 8, 256, 128) == 0
