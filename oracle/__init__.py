"""CPU fp64 oracle for the MISA indexer path -- test infrastructure only.

Imported by the tests, the package smoke check and the benchmark's CPU-baseline
leg; never by the product path.
"""

from .misa_oracle import *  # noqa: F401,F403
