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
