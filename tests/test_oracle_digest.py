"""The oracle's outputs on a fixed small workload match the digests stored
by tests/golden/make_oracle_digest.py (guards against unintended changes of
the oracle's arithmetic)."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))


def test_oracle_digest_unchanged(orc):
    import make_oracle_digest as m

    stored = [l.strip() for l in open(m.OUT) if l.strip() and not l.startswith("#")]
    assert m.lines() == stored
