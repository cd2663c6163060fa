"""The CPU oracle against its pins (no GPU)."""
import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin_single_thread(orc, pin):
    pin(orc)


@pytest.mark.parametrize("pin", [oracle_pins.pin_c_vs_numpy, oracle_pins.pin_linear,
                                 oracle_pins.pin_scale_closed_form], ids=lambda f: f.__name__)
def test_pin_openmp_build(orc_omp, pin):
    pin(orc_omp)
