"""Plant plausible mistakes in copies of the oracle and check the pins catch
every one of them (each planted copy must fail at least one pin)."""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

PLANTS = {
    1: "rel index sign flipped (kh - qh instead of qh - kh)",
    2: "rel_w term dropped",
    3: "Rh and Rw swapped",
    4: "patch grid read transposed",
    5: "scale applied to the rel-pos bias",
    6: "GQA kv head tiled (h % Hkv) instead of repeated (h / g)",
    7: "causal diagonal excluded",
    8: "sliding window one key too wide",
    10: "softmax not normalised",
    11: "float mask batch stride ignored",
    12: "boolean mask polarity inverted",
    13: "rel index shifted by the query grid size instead of the key grid size",
}


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=lambda p: f"plant{p}")
def test_planted_mistake_is_caught(plant, tmp_path):
    path = oracle.compile_oracle(str(tmp_path / f"liboracle_plant{plant}.so"), plant=plant)
    lib = oracle.load(path)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except Exception:  # an assertion, or a planted copy rejecting its inputs
            failed.append(pin.__name__)
    assert failed, f"no pin caught planted mistake {plant}: {PLANTS[plant]}"
