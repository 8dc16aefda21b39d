"""Exact fused scaled-dot-product attention for NVIDIA B200 (sm_100a).

    from exact_attention_sdpa_b200 import attn_fwd, attn_bwd
    out, lse = attn_fwd(q, k, v, causal=True)           # also: bias=, gate=, softcap=, ...
    dq, dk, dv = attn_bwd(q, k, v, out, lse, dout, causal=True)

Ragged batches: ``attn_fwd_varlen``; 8-bit (e4m3) inputs: ``attn_fwd_fp8``; host
buffers end to end: ``fwd`` (with ``Staging``).

The computation runs in ``libattn.so`` (built in-tree by
``python -m exact_attention_sdpa_b200.build``); this package only marshals
arguments.  Importing it does not load the library; the first call does, and
raises if the library is missing.
"""
from ._native import (AttnError, Staging, attn_bwd, attn_fwd, attn_fwd_fp8, attn_fwd_raw, attn_fwd_varlen, fwd,
                      last_device_status, load_library, set_wait_limit, status_string, version)

__all__ = ["attn_fwd", "attn_bwd", "attn_fwd_varlen", "attn_fwd_fp8", "attn_fwd_raw", "fwd", "Staging", "AttnError", "last_device_status", "load_library",
           "set_wait_limit", "status_string", "version"]
