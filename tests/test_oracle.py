"""The oracle against its pins (CPU only), and planted mistakes against the pins."""
import os
import tempfile

import numpy as np
import pytest

import oracle as oracle_mod
from pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(oracle, pin):
    pin(oracle)


_PLANT_DIR = tempfile.mkdtemp(prefix="prism_ref_plants_")


@pytest.mark.parametrize("plant", sorted(oracle_mod.PLANTS))
def test_planted_mistake_is_caught(plant):
    """Each deliberately wrong oracle build must fail at least one pin."""
    o = oracle_mod.load(plant=plant, out_dir=_PLANT_DIR)
    assert o.plant == plant
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except AssertionError:
            failed.append(pin.__name__)
        except (ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"plant {plant} ({oracle_mod.PLANTS[plant]}) passed every pin"


def test_decode_step_rejects_bad_arguments(oracle):
    q = np.zeros((2, 1, 4, 8), np.uint16)
    k = [np.zeros((1, 2, 16, 8), np.uint16)] * 2
    lens = np.array([16], np.int32)
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, k, lens, 4, 1, [0, 1])          # layer 0 not an anchor
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, k, np.array([17], np.int32), 4, 1, [1, 0])   # len > Lmax
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, k, lens, 4, -1, [1, 0])         # negative radius
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, k, lens, 4, 1, [2, 0])          # layer 0 shared
    with pytest.raises(ValueError):
        oracle.decode_step(q, k, k, lens, 4, 1, [1, 3])          # unknown layer kind
    out, idx = oracle.decode_step(q, k, k, np.array([0], np.int32), 4, 1, [1, 0])
    assert np.all(idx == -1) and np.all(out == 0.0), "empty context: nothing selected"


def test_oracle_build_is_threaded():
    assert oracle_mod.load().num_threads() >= 1
    assert os.path.exists(oracle_mod.load().path)
