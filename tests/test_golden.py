"""The oracle reproduces its committed regression fixtures (tests/golden/,
written by tests/golden/make_golden.py from the oracle alone): a change to the
oracle's arithmetic shows here and must regenerate them deliberately."""
import json
import os

import numpy as np
import pytest

from .golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(scope="module")
def stored():
    with open(os.path.join(HERE, "tiny_layer.json")) as f:
        return json.load(f)["values"]


def test_oracle_reproduces_its_fixtures(stored):
    now = make_golden.compute()
    assert sorted(now) == sorted(stored)
    for k in stored:
        np.testing.assert_allclose(np.asarray(now[k]), np.asarray(stored[k]), rtol=1e-13,
                                   atol=1e-15, err_msg=k)
