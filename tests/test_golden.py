"""The oracle against its committed fixture (tests/golden/tiny_w4a4.json,
written by tests/golden/make_golden.py from the oracle alone): a change to the
oracle's arithmetic or to the input generator shows up here."""
import json
import os

from tests.golden.make_golden import compute

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_w4a4.json")


def test_oracle_matches_golden_fixture():
    with open(HERE) as f:
        stored = json.load(f)
    assert compute() == stored
