"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.PINS, ids=[p.__name__ for p in pins.PINS])
def test_pin(pin):
    pin(oracle.default())


def test_oracle_rejects_bad_lengths():
    q, r, k, v, _ = pins.rand_case(0)
    with pytest.raises(ValueError):
        oracle.parallax_decode(q, r, k, v, [25, 3], 0.3)  # 25 > Lmax = 24
    with pytest.raises(ValueError):
        oracle.parallax_decode(q, r, k, v, [-1, 3], 0.3)
