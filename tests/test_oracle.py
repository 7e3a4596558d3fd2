"""The CPU oracle against its pins (no GPU).  See tests/oracle_pins.py."""
import pytest

from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


from oracle_pins import AM_PINS  # noqa: E402


@pytest.mark.parametrize("pin", AM_PINS, ids=[p.__name__ for p in AM_PINS])
def test_oracle_am_pin(pin):
    import oracle.datafree_am as am
    pin(am)


from oracle_pins import LORA_PINS  # noqa: E402


@pytest.mark.parametrize("pin", LORA_PINS, ids=[p.__name__ for p in LORA_PINS])
def test_oracle_lora_pin(pin):
    import oracle.lora_backward as lb
    pin(lb)
