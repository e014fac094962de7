"""fp64 CPU oracle for the DoSA indexer.  Test infrastructure: imported only by
tests/, __graft_entry__.smoke() and bench.py's CPU-baseline legs."""
from .dosa_oracle import *  # noqa: F401,F403
