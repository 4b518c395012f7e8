"""The fp64 oracle against facts fixed outside it (runs on CPU)."""
import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin, lib):
    pin(lib)


def test_no_rescale_streamer_is_wrong():
    # FlashAttention, Playable, EP 04: skipping the rescale is wrong by 40% or more
    # once a later tile brings a bigger max.
    assert oracle_pins.check_no_rescale_fails() > 0.4


def test_oracle_rejects_bad_rows(lib):
    import numpy as np
    q = np.zeros((1, 1, 4, 2), np.float32)
    with pytest.raises(RuntimeError):
        oracle.attention_fwd(q, q, q, 1.0, False, rows=np.array([[[4]]]), lib=lib)
