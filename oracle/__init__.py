"""Float64 CPU oracle of the POET-X layer.

TEST INFRASTRUCTURE: only the tests, the package entry point's smoke check and
the benchmark's CPU-baseline leg may import this package.  The product path
never does.
"""
from .poetx_oracle import *  # noqa: F401,F403
