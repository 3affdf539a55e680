"""Regression check of the oracle against its stored outputs on the tiny decode batch.

The fixture was written by tests/golden/make_golden.py, which calls only the oracle: it
detects later changes to the oracle's results, it does not pin the oracle."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))


def test_oracle_matches_stored_tiny_decode_outputs():
    import make_golden
    rec = json.load(open(os.path.join(HERE, "golden", "tiny_decode_oracle.json")))
    out, digest = make_golden.compute()
    assert digest == rec["inputs_sha256"], "the seeded inputs changed"
    assert list(out.shape) == rec["shape"]
    assert np.allclose(out.reshape(out.shape[0], -1), np.array(rec["rows"]), atol=1e-11, rtol=0)
