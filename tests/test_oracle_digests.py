"""The oracle's outputs on the seeded cases of tests/golden/make_oracle_digests.py
are the ones stored in tests/golden/oracle_digests.json: a change of the
oracle's arithmetic shows up here and must be regenerated on purpose."""
import json
import os

from tests.golden.make_oracle_digests import digests

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_outputs_match_the_stored_digests():
    stored = json.load(open(os.path.join(HERE, "golden", "oracle_digests.json")))["cases"]
    assert digests() == stored
