"""The fp64 oracle against its pins (no GPU)."""
import pytest

from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_golden_regression():
    """The oracle still reproduces tests/golden/small_case.json (written by make_golden.py)."""
    import json
    import os

    import numpy as np

    import oracle
    path = os.path.join(os.path.dirname(__file__), "golden", "small_case.json")
    doc = json.load(open(path))
    inp = {k: (np.array(v) if v is not None else None) for k, v in doc["inputs"].items()}
    out, sf = oracle.recurrent(**inp)
    assert np.max(np.abs(out - np.array(doc["out"]))) < 1e-12
    assert np.max(np.abs(sf - np.array(doc["final_state"]))) < 1e-12
