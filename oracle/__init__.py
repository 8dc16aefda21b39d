"""fp64 CPU oracle (test infrastructure only; see oracle/sdpa.py)."""
from .sdpa import sdpa_backward, sdpa_forward, sdpa_rows, sdpa_varlen_forward, to_f64

__all__ = ["sdpa_forward", "sdpa_rows", "sdpa_backward", "sdpa_varlen_forward", "to_f64"]
