"""The oracle still produces the stored tiny-workload fixture.

tests/golden/tiny_oracle.json is written by tests/golden/make_golden.py,
which calls only the oracle and the seeded input generator; a change to the
oracle's arithmetic that moves these values must regenerate the fixture and
name, in its commit message, the passage that justifies the change.
"""

import json
import os

from tests.golden.make_golden import compute

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_fixture_unchanged():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        want = json.load(f)
    got = json.loads(json.dumps(compute()))
    assert got == want
