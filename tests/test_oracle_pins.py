"""The fp64 oracle against the facts that pin it (see ``oracle_pins.py``)."""
import pytest

from oracle_pins import PINS


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


def test_oracle_rejects_bad_arguments(orc):
    import numpy as np
    Q = np.zeros((1, 3, 2, 4))
    K = np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):
        orc.attn_fwd(Q, K, K, 1.0)                       # Hq % Hkv != 0
    Q = np.zeros((1, 2, 2, 4))
    with pytest.raises(ValueError):
        orc.attn_fwd(Q, K, K, 1.0, causal=False, window=2)  # window needs causal
    with pytest.raises(ValueError):
        orc.decode(np.zeros((1, 2, 4)), K, K, np.array([3]))  # length above capacity
