"""The oracle's layout derivation and references (re-exported for the tests)."""
from oracle.workload import OLayout, assert_same_layout, groups, layout, reference, retained  # noqa: F401
