"""fp64 CPU oracle for indexed sparse decode attention -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg use it;
the library never does.
"""

from . import lisa_oracle  # noqa: F401
