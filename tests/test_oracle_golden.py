"""The oracle against its stored outputs (tests/golden/oracle_tiny.json, written
by tests/golden/make_golden.py, which calls only the oracle): a regression
guard, so that a change of the oracle's arithmetic is a visible, deliberate
diff.  The independent pins of the same functions are in
test_oracle_formats.py and test_oracle_attention.py."""
import json
import os

import numpy as np

from tests.golden import make_golden


def test_oracle_matches_stored_outputs():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny.json")
    stored = json.load(open(path))
    now = make_golden.compute()
    assert stored["shape"] == now["shape"] and stored["rows"] == now["rows"]
    for a, b in zip(stored["cases"], now["cases"]):
        assert (a["fmt"], a["mode"], a["tau"]) == (b["fmt"], b["mode"], b["tau"])
        np.testing.assert_allclose(np.array(b["O"]), np.array(a["O"]), rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(np.array(b["lse"]), np.array(a["lse"]), rtol=1e-12)
