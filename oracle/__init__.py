"""fp64 CPU oracle of the MLA layer.  Test infrastructure: imported only by
tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg."""
