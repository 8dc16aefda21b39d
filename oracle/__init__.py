"""fp64 CPU oracle (test infrastructure only; see oracle/sdpa.py and oracle/fp8.py)."""
from .fp8 import e4m3_decode, e4m3_encode, e4m3_round, p_rounding_bound, sdpa_forward_fp8
from .sdpa import sdpa_backward, sdpa_forward, sdpa_rows, sdpa_varlen_forward, to_f64

__all__ = ["sdpa_forward", "sdpa_rows", "sdpa_backward", "sdpa_varlen_forward", "to_f64",
           "e4m3_decode", "e4m3_encode", "e4m3_round", "sdpa_forward_fp8", "p_rounding_bound"]
