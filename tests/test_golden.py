"""The oracle still reproduces its recorded output on the small golden case."""
import json
import os

import numpy as np

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")


def test_oracle_matches_golden_record():
    with open(HERE) as f:
        ref = json.load(f)
    got = make_golden.compute()
    assert got["case"] == ref["case"]
    assert got["idx"] == ref["idx"]
    assert np.allclose(got["o_row_sums"], ref["o_row_sums"], rtol=0, atol=1e-5)
    assert np.allclose(got["lse"], ref["lse"], rtol=0, atol=1e-5)
    assert np.allclose(got["pyramid_top"], ref["pyramid_top"], rtol=0, atol=1e-6)
