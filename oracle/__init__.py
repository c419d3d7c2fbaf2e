"""fp64 CPU oracle for the SLA hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package; the product path never does.
"""
from .sla_oracle import *  # noqa: F401,F403
from .sla_oracle import __all__  # noqa: F401
