"""fp64 CPU oracle of the STCA forward pass.  Test infrastructure only: imported by
tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and reference legs,
never by the product path."""
from . import stca_oracle  # noqa: F401
