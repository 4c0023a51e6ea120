"""fp64 CPU oracle of the DLRM hot path. Test infrastructure only (see oracle.py)."""
