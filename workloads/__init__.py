"""Seeded synthetic inputs for indexed sparse decode attention.

This package only draws random numbers and lays them out in the cache
formats the library reads.  It is shared by the tests, the benchmark and the
smoke check; it holds none of the decode path's arithmetic (no averaging of
the query group for scoring, no top-M, no attention, no linear-branch update).
"""

from .synth import (  # noqa: F401
    DecodeProblem,
    LayeredProblem,
    LinearBranchInputs,
    make_problem,
    config1,
    config2,
    config3,
    config4,
    config5,
    CONFIG_NAMES,
)
