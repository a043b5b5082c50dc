"""The oracle against values and routines it does not share code with (CPU only)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(o, check):
    check(o)


def test_golden_file_has_the_two_worked_values():
    rows = oracle_pins.golden_kv_bytes()
    assert rows[0][-1] == 2 * 1024 ** 3      # 2 GiB with 32 KV heads
    assert rows[1][-1] == 512 * 1024 ** 2    # 512 MiB with 8 KV heads
