"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This package only draws random numbers and lays out shapes: model weights,
prefix tokens, draft-tree shapes and the planting draws.  It contains none of
the arithmetic of tree verification; the planting helper takes the target's
argmax from a caller-supplied function (the float64 oracle in the tests, the
library in the benchmark).
"""

from .workloads import *  # noqa: F401,F403
