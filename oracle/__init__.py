"""CPU oracle for the LSA indexer and sparse attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline / reference legs import this package; the library
(`hierarchical_key_clustering_b200`) never does, and the two share no code.
"""
from .oracle import *  # noqa: F401,F403
