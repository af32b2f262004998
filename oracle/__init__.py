"""fp64 CPU oracle (test infrastructure only; see attn_ref.py)."""
