"""Failure detection without a GPU fault: every mbarrier wait in the kernel is
bounded.  The injected stall makes the MMA warp wait on a barrier nothing
arrives on; after the wait budget the kernel records a timeout in its status
word, every role drains its in-flight copies and MMAs and the kernel exits;
the context stays usable and the next normal call is correct."""
import pytest
import torch

from exact_attention_sdpa_b200 import _native as nat
from exact_attention_sdpa_b200 import attn_fwd, last_device_status, set_wait_limit
from exact_attention_sdpa_b200.workloads import Workload, make_inputs
from oracle import sdpa_forward
from helpers import assert_close_to_oracle

DEFAULT_LIMIT = 1 << 32


@pytest.mark.gpu
def test_timeout_is_reported_and_context_survives():
    w = Workload("st", B=2, H=4, N=1024, d=64, dtype="fp16", causal=True, seed=5)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    assert last_device_status() == nat.ATTN_OK          # clears any stale word
    try:
        set_wait_limit(1 << 21)                          # ~1 ms per bounded wait
        nat.debug_inject_stall(True)
        attn_fwd(q, k, v, causal=True, scale=w.scale)
        assert last_device_status() == nat.ATTN_ERR_TIMEOUT
    finally:
        nat.debug_inject_stall(False)
        set_wait_limit(DEFAULT_LIMIT)
    assert last_device_status() == nat.ATTN_OK          # the word was cleared by the read
    o, lse = attn_fwd(q, k, v, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert last_device_status() == nat.ATTN_OK
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], causal=True, scale=w.scale)
    assert_close_to_oracle(o, lse, o_ref, l_ref, torch.float16, "after-timeout")


VARIANTS = {
    # the same stall and abort path in the other kernel builds: staged pair bias + gate at d = 32,
    # P inside S at d = 128, and the score-modification build (softcap + left window)
    "d32_bias_gate": (Workload("st32", B=2, H=2, N=300, d=32, dtype="bf16", causal=False, seed=6, bias=True,
                               gate=True), {}),
    "d128_causal": (Workload("st128", B=1, H=2, N=600, d=128, dtype="bf16", causal=True, seed=7), {}),
    "d64_mods": (Workload("stm", B=1, H=2, N=700, d=64, dtype="fp16", causal=True, seed=8),
                 {"softcap": 20.0, "window_left": 150}),
}


@pytest.mark.gpu
@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_timeout_in_other_builds(variant):
    from helpers import padded
    w, mods = VARIANTS[variant]
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    bias = None if inp["bias"] is None else padded(inp["bias"], dev)
    gate = None if inp["gate"] is None else inp["gate"].to(dev)
    assert last_device_status() == nat.ATTN_OK
    try:
        set_wait_limit(1 << 21)
        nat.debug_inject_stall(True)
        attn_fwd(q, k, v, bias=bias, gate=gate, causal=w.causal, scale=w.scale, **mods)
        assert last_device_status() == nat.ATTN_ERR_TIMEOUT
    finally:
        nat.debug_inject_stall(False)
        set_wait_limit(DEFAULT_LIMIT)
    o, lse = attn_fwd(q, k, v, bias=bias, gate=gate, causal=w.causal, scale=w.scale, **mods)
    torch.cuda.synchronize()
    assert last_device_status() == nat.ATTN_OK
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], bias=inp["bias"], gate=inp["gate"], causal=w.causal,
                                scale=w.scale, **mods)
    assert_close_to_oracle(o, lse, o_ref, l_ref, w.torch_dtype, f"after-timeout {variant}")


def test_wait_limit_setter_is_host_only():
    # host-side setter; no device work (runs without a GPU)
    nat.load_library()
    set_wait_limit(5)            # raised to the 1024-cycle floor internally
    set_wait_limit(DEFAULT_LIMIT)
