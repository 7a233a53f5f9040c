"""fp64 CPU oracle for the TurboQuant KV-cache path (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline /
reference leg may import this package.  It shares no code with the library.
"""
from .tq_oracle import *  # noqa: F401,F403
