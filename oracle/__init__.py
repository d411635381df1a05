"""Plain fp64 CPU oracle of the ReSA decode hot path (test infrastructure).

Only the tests, the graft entry point's smoke check and the CPU-baseline leg of
the benchmark may import this package; the library itself never does.
"""
from .resa_oracle import *  # noqa: F401,F403
