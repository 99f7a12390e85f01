"""The oracle's outputs on the five seeded workloads still hash to the committed
digests (tests/golden/digests.json, written by tests/golden/make_golden.py).
A change here means the oracle's arithmetic or the input generator changed."""
import json
import os

import pytest

from tests.golden.make_golden import FULL, SAMPLED, digests

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "digests.json")))


@pytest.mark.parametrize("name", FULL + SAMPLED)
def test_oracle_digests(name):
    assert digests(name) == GOLD[name]
