"""The oracle's output on the tiny seeded layer must not drift silently (CPU only).

A change here means the oracle's arithmetic or the generator changed; the
commit that regenerates the digest must name the passage that justifies it.
"""
import os
import sys

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
import make_oracle_digest  # noqa: E402


def test_oracle_tiny_digest_unchanged():
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny_digest.txt")
    assert make_oracle_digest.digest() == open(path).read()
