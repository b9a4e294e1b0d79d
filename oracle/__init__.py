"""fp64 CPU oracle -- test infrastructure only (see mmdit_oracle.py).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package; the product path never does.
"""
from .mmdit_oracle import *  # noqa: F401,F403
