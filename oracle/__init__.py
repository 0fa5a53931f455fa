"""fp64 CPU oracle for the tile-sparse attention path (test infrastructure only).

Only the tests, the smoke check and the bench's CPU-baseline leg use it; the
product path never imports it.
"""
from . import veda_oracle  # noqa: F401
