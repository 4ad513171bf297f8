"""fp64 CPU oracle of the MTA forward pass -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py may
import this package.  The library never does.
"""
from .mta_oracle import *  # noqa: F401,F403
from .mta_oracle import __all__  # noqa: F401
