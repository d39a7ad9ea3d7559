"""The fp64 oracle against its pins (CPU only)."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.FAST_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_needles_8k_selected(orc):
    pins.pin_needles_selected(orc, "8k")


def test_score_sums_on_full_8k(orc):
    from block_sparse_attention_27_b200 import workloads as W
    pins.pin_score_sums(orc, W.make("8k", 0))
