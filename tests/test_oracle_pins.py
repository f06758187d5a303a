"""The fp64 oracle against closed forms, invariants, brute force and torch SDPA."""
import pytest

import oracle
from oracle_pins import ALL_PINS, pin_torch_sdpa_large_slice


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle.lib())


def test_pin_large_slice():
    pin_torch_sdpa_large_slice(oracle.lib())


def test_rejects_bad_shapes():
    import numpy as np
    z = np.zeros((1, 2, 1, 4))
    with pytest.raises(ValueError):
        oracle.attention_f64(z, z, np.zeros((1, 3, 1, 4)), 1.0)
    bits = np.zeros((1, 4, 3, 2, 8), dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.attention_rows_packed_bf16(bits, 1.0, [(0, 2, 0)])


def test_empty_batch():
    import numpy as np
    z = np.zeros((0, 5, 2, 8))
    assert oracle.attention_f64(z, z, z, 1.0).shape == (0, 5, 2, 8)
