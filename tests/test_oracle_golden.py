"""The oracle reproduces its stored tiny-case values (tests/golden/oracle_tiny.json, written
by tests/golden/make_golden.py from the oracle alone).  Guards against unintended changes."""
import json
import os

import numpy as np

from tests.golden import make_golden


def test_oracle_matches_stored_tiny_case():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny.json")
    stored = json.load(open(path))
    now = make_golden.compute()
    assert stored["case"] == now["case"]
    for case in ("mc0", "mc1", "terms", "exact", "packed"):
        for key in now[case]:
            assert np.allclose(np.array(stored[case][key]), np.array(now[case][key]), rtol=1e-13, atol=1e-15), \
                (case, key)
