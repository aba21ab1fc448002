"""The oracle's output on small seeded workloads equals the committed digests
(tests/golden/oracle_digests.json, written by tests/golden/make_golden.py from the oracle only)."""
import json
import os
import sys

import pytest

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
import make_golden  # noqa: E402

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_digests.json")))


@pytest.mark.parametrize("case", make_golden.CASES, ids=[c[0] for c in make_golden.CASES])
def test_oracle_matches_frozen_digest(case):
    assert make_golden.digest(case) == GOLD[case[0]]


@pytest.mark.parametrize("case", make_golden.DENSE_CASES, ids=[c[0] for c in make_golden.DENSE_CASES])
def test_dense_oracle_matches_frozen_digest(case):
    assert make_golden.digest_dense(case) == GOLD[case[0]]
