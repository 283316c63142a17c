"""The oracle still reproduces its stored regression fixtures exactly."""
import json
import os

import pytest

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", ["oracle_c8p3_12x50", "oracle_c12p4_10x61"])
def test_oracle_matches_golden(oracle_mod, name):
    import sys
    sys.path.insert(0, HERE)
    from make_golden import CASES, case_values
    with open(os.path.join(HERE, name + ".json")) as fh:
        stored = json.load(fh)
    case = [c for c in CASES if c[0] == name][0]
    now = case_values(*case[1:])
    for k in ("fmt", "W_row0", "W_sum", "y", "yabs"):
        assert now[k] == stored[k], k
