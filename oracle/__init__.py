"""Float64 CPU oracle -- test infrastructure only (see la_oracle.py).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package.  It shares no code with the CUDA library.
"""
