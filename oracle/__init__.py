"""fp64 CPU oracle (test infrastructure only; see osdn_ref.py)."""
