"""Stored oracle digests (written by tests/golden/make_golden.py, which calls
only the oracle) still match: guards the oracle against silent drift."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))


def test_oracle_digests_unchanged(oracle_mod):
    import make_golden

    stored = json.load(open(os.path.join(HERE, "golden", "oracle_digests.json")))
    assert make_golden.compute() == stored
