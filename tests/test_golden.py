"""The oracle still reproduces its frozen golden values (tests/golden)."""
import json
import os

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_matches_frozen_golden():
    with open(os.path.join(HERE, "tiny_f32_oracle.json")) as fh:
        ref = json.load(fh)
    now = make_golden.compute()
    assert now["out"] == ref["out"]
    assert now["last_state"] == ref["last_state"]
