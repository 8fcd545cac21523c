"""CPU oracle (test infrastructure only; see dsa_ref.py)."""
