"""The oracle against its pins (CPU only)."""
import pytest

import oracle
from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle.default())


def test_bad_arguments_rejected():
    import torch
    q = torch.zeros(1, 3, 8)
    k = torch.zeros(4, 2, 8)
    with pytest.raises(ValueError):
        oracle.attn(q, k, k, [4], 3, 2, 1.0)      # h_q not a multiple of h_kv
    with pytest.raises(ValueError):
        oracle.attn(q[:, :2], k, k, [-1], 2, 2, 1.0)  # negative length
