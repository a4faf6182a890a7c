"""fp64 CPU oracle for ReHyAt chunked hybrid attention -- test infrastructure.

Only tests/, __graft_entry__.smoke() and bench.py (cpu_baseline leg and the
--impl reference arm) may import this package.  It shares no code with the CUDA
library and imports nothing from it.
"""
from .rehyat_oracle import *  # noqa: F401,F403
