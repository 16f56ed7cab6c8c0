"""The backward oracle against its pins (tests/oracle_bwd_pins.py)."""
import pytest

import oracle
import oracle_bwd_pins


@pytest.mark.parametrize("name", list(oracle_bwd_pins.ALL_PINS))
def test_pin(name):
    ok, detail = oracle_bwd_pins.ALL_PINS[name](oracle.attn_jvp_bwd)
    assert ok, f"{name}: {detail}"


def test_bad_arguments_rejected():
    import numpy as np
    x = np.zeros((1, 2, 4))
    with pytest.raises(RuntimeError):
        oracle.attn_jvp_bwd(x, x, x, x, x, x, x, x, 0.5, qrows=[2])  # row out of range
    with pytest.raises(RuntimeError):
        oracle.attn_jvp_bwd(x, x, x, x, x, x, x, x, 0.5, krows=[-1])
