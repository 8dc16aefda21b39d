"""GPU parity of the score modifications (attn_fwd_ex: ALiBi, logit softcap,
left window) against the fp64 oracle on the same seeded inputs, every output
row compared, with the forward's tolerances."""

import pytest
import torch

from exact_attention_sdpa_b200 import attn_fwd, last_device_status
from exact_attention_sdpa_b200.workloads import Workload, make_inputs
from oracle import sdpa_forward
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu


def _alibi_slopes(h):
    # the usual geometric sequence 2^(-8 (i+1) / H); any per-head values would do
    return torch.tensor([2.0 ** (-8.0 * (i + 1) / h) for i in range(h)], dtype=torch.float32)


CASES = [  # N, Nk, d, causal, dtype, softcap, alibi, window
    (300, 300, 64, True, "fp16", 2.0, False, -1),
    (257, 257, 128, False, "bf16", 0.0, True, -1),
    (400, 400, 32, True, "bf16", 0.0, False, 100),
    (300, 700, 64, True, "bf16", 1.5, True, 200),
    (640, 640, 64, True, "fp16", 3.0, True, 0),
    (129, 300, 128, False, "fp16", 1.0, False, 50),     # softcaps of 1-3 bend N(0,1) scores visibly
    (1000, 1000, 64, True, "bf16", 0.0, True, 383),
]


@pytest.mark.parametrize("N,Nk,d,causal,dtype,softcap,alibi,window", CASES)
def test_score_modifications(N, Nk, d, causal, dtype, softcap, alibi, window):
    H = 4
    # inputs N(0,1) as everywhere: the stated tolerances are for outputs of that scale
    w = Workload("mods", B=2, H=H, N=N, d=d, dtype=dtype, causal=causal, seed=80 + N % 7, Nk=Nk)
    inp = make_inputs(w)
    slopes = _alibi_slopes(H) if alibi else None
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o, lse = attn_fwd(q, k, v, causal=causal, scale=w.scale, softcap=softcap,
                      alibi_slopes=None if slopes is None else slopes.to(dev), window_left=window)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], causal=causal, scale=w.scale, softcap=softcap,
                                alibi_slopes=slopes, window_left=window)
    assert_close_to_oracle(o, lse, o_ref, l_ref, w.torch_dtype, f"mods N={N} Nk={Nk} d={d}")


def test_no_modification_is_the_plain_forward():
    w = Workload("mods0", B=1, H=2, N=333, d=64, dtype="fp16", causal=True, seed=88)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o0, l0 = attn_fwd(q, k, v, causal=True, scale=w.scale)
    o1, l1 = attn_fwd(q, k, v, causal=True, scale=w.scale, window_left=10**6)   # a window wider than N
    torch.cuda.synchronize()
    assert torch.equal(l0, l1) or torch.allclose(l0, l1, atol=1e-6)
    assert (o0.float() - o1.float()).abs().max().item() <= 1e-3


def test_window_workload_full_size_sampled():
    """The benchmarked sliding-window workload (N=8192, a 1024-key left window, causal): the
    kernel skips the key tiles left of each unit's window.  Sampled rows of four heads and
    every row of one whole head are compared with the oracle."""
    import numpy as np
    from exact_attention_sdpa_b200.workloads import WORKLOADS
    from oracle import sdpa_rows
    w = WORKLOADS["n8192_window"]
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o, lse = attn_fwd(q, k, v, causal=True, scale=w.scale, window_left=w.window_left)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    rng = np.random.default_rng(3)
    picks = []
    for b, h in [(0, 0), (w.B - 1, w.H - 1), (1, 5), (2, 7)]:
        rows = {0, 1, 127, 128, 255, 256, 1023, 1024, 1025, 1151, 1152, 4095, 4096, w.N - 1}
        rows.update(int(x) for x in rng.integers(0, w.N, size=20))
        picks += [(b, h, i) for i in sorted(rows)]
    o_ref, l_ref = sdpa_rows(inp["q"], inp["k"], inp["v"], picks, causal=True, scale=w.scale,
                             window_left=w.window_left)
    idx = tuple(np.array(x) for x in zip(*picks))
    assert_close_to_oracle(o.cpu()[idx], lse.cpu()[idx], o_ref, l_ref, w.torch_dtype, "n8192_window sampled")
    sl = (slice(3, 4), slice(11, 12))
    o_ref, l_ref = sdpa_forward(inp["q"][sl], inp["k"][sl], inp["v"][sl], causal=True, scale=w.scale,
                                window_left=w.window_left)
    assert_close_to_oracle(o.cpu()[sl], lse.cpu()[sl], o_ref, l_ref, w.torch_dtype, "n8192_window head (3,11)")


WINDOW_CASES = [  # N, Nk, d, causal, window: ranges that skip many key tiles, ragged offsets
    (1500, 1500, 64, True, 130),
    (700, 2900, 128, True, 257),
    (900, 900, 32, False, 300),       # without causal masking: keys from i - w to the end
    (333, 1400, 64, False, 1),
    (700, 2900, 64, True, 129),       # the second query tile of most units starts a key tile later
    (1300, 1300, 32, True, 511),
]


@pytest.mark.parametrize("N,Nk,d,causal,window", WINDOW_CASES)
def test_window_tile_skipping(N, Nk, d, causal, window):
    w = Workload("win", B=1, H=3, N=N, d=d, dtype="bf16", causal=causal, seed=95 + window % 5, Nk=Nk)
    inp = make_inputs(w)
    dev = torch.device("cuda")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o, lse = attn_fwd(q, k, v, causal=causal, scale=w.scale, window_left=window)
    torch.cuda.synchronize()
    assert last_device_status() == 0
    o_ref, l_ref = sdpa_forward(inp["q"], inp["k"], inp["v"], causal=causal, scale=w.scale, window_left=window)
    assert_close_to_oracle(o, lse, o_ref, l_ref, torch.bfloat16, f"window {window} N={N} Nk={Nk}")
