"""The oracle's decode trajectories on the tiny configuration against the
stored record (tests/golden/oracle_trajectories.json, written by
tests/golden/make_oracle_trajectories.py from the oracle alone): any change
of the oracle's arithmetic or drivers shows up here and must be recorded
anew with its justification."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_oracle_trajectories as M  # noqa: E402


def test_oracle_trajectories_match_the_record():
    with open(M.OUT) as f:
        want = json.load(f)
    got = M.trajectories()
    assert got == want
    # the structural facts the record also shows
    assert got["spec_linear"] == got["ar"] == got["spec_quadratic"]
    assert got["routing_k1_passes"][2] == got["routing_k2_passes"][2] == 3      # one causal append per block
